"""Shared test helpers: moving tensors between torch and the oracle's numpy
arrays, and the tolerance check.  No arithmetic of the method here."""
import numpy as np
import torch


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 / int16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u32(t: torch.Tensor) -> np.ndarray:
    """uint8 byte buffer -> numpy uint32 words (host copy)."""
    return t.detach().contiguous().cpu().numpy().view(np.uint32)


def w_np(W: torch.Tensor) -> np.ndarray:
    """Weights for the oracle: fp32 as is, bf16 as uint16 bit patterns."""
    if W.dtype == torch.bfloat16:
        return u16(W)
    return W.detach().contiguous().cpu().numpy()


def assert_within(y_gpu: torch.Tensor, y64: np.ndarray, yabs: np.ndarray, out: str, oracle, what: str = ""):
    """|y - y_ref| <= 1e-5 sum|x w| (+ 4e-3 |y_ref| for bf16 outputs).

    fp32 outputs are compared with the oracle's fp32 rounding of the exact
    sum.  bf16 outputs are compared with the exact sum itself: the 4e-3
    relative allowance is there to cover one bf16 rounding (at most 2^-8
    relative), and measuring from the oracle's own bf16 rounding would count
    that rounding twice (a result on the other side of a rounding boundary
    is one bf16 ulp, up to 2^-7 relative, from it)."""
    ref = np.asarray(y64, dtype=np.float64) if out == "bf16" else oracle.round_out(y64, out)
    got = y_gpu.detach().float().cpu().numpy().astype(np.float64)
    tol = oracle.tolerance(ref, yabs, out)
    err = np.abs(got - ref.astype(np.float64))
    bad = np.nonzero(~(err <= tol))[0] if err.ndim == 1 else np.argwhere(~(err <= tol))
    assert bad.size == 0, (f"{what}: {len(bad)} outputs out of tolerance; first {bad[:5].tolist()}, "
                           f"err {err.reshape(-1)[:3]}, tol {tol.reshape(-1)[:3]}")
    return float((err / np.maximum(tol, 1e-300)).max()) if err.size else 0.0
