"""Thin Python binding of libtb_b200.so (include/tb.h).

Argument marshalling only: tensors are passed as raw device pointers with
the current CUDA stream of their device; every computation runs in the
library's kernels.  There is no host fallback: if the shared library is
missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libtb_b200.so")

TERNARY, INT2, INT3 = 0, 1, 2
TERNARY_B3 = 3  # the ternary grid, 5 codes per byte
F32, BF16 = 0, 1
MAX_LAYER_ITEMS = 16
FLAG_OVERLAP_PREVIOUS = 1
FLAG_TEST_STALL = 0x80000000  # test hook: the batch-1 kernel's waits give up (see include/tb.h)
NOALLOC_SCRATCH_BYTES = 4 << 20  # TB_NOALLOC_SCRATCH_BYTES

STATUS = {0: "TB_OK", 1: "TB_ERR_ARG", 2: "TB_ERR_SHAPE", 3: "TB_ERR_ALIGN", 4: "TB_ERR_UNSUPPORTED", 5: "TB_ERR_CUDA",
          6: "TB_ERR_TIMEOUT"}

# every entry point the header declares: (name, restype, argtypes)
_P, _I64, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "tb_version": (ctypes.c_int, []),
    "tb_status_string": (ctypes.c_char_p, [_I32]),
    "tb_packed_bytes": (_SZ, [_I32, _I64, _I64]),
    "tb_scale_bytes": (_SZ, [_I64, _I64]),
    "tb_scales_absmax": (_I32, [_P, _I32, _I64, _I64, _I32, _P, _P]),
    "tb_pack": (_I32, [_P, _I32, _I64, _I64, _I32, _P, _P, _P, _P]),
    "tb_unpack": (_I32, [_P, _I32, _I64, _I64, _P, _P]),
    "tb_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "tb_layer_workspace_bytes": (_SZ, [_P, _I32]),
    "tb_gemv": (_I32, [_P, _I32, _P, _P, _P, _I32, _I64, _I64, _P, _SZ, _P]),
    "tb_gemm": (_I32, [_P, _I32, _P, _P, _I64, _P, _I32, _I64, _I64, _I64, _I64, _P, _SZ, _P]),
    "tb_layer_gemv": (_I32, [_P, _I32, ctypes.c_uint, _P, _SZ, _P]),
    "tb_gemv_noalloc": (_I32, [_P, _I32, _P, _P, _P, _I32, _I64, _I64, _P]),
    "tb_wait_timeouts": (ctypes.c_uint, []),
    "tb_sync_status": (_I32, [_P]),
    "tb_gate_up_workspace_bytes": (_SZ, [_P, _P]),
    "tb_gate_up_silu": (_I32, [_P, _P, _P, ctypes.c_uint, _P, _SZ, _P]),
}


class Linear(ctypes.Structure):
    """tb_linear_t"""
    _fields_ = [("packed", _P), ("scales", _P), ("x", _P), ("y", _P), ("N", _I64), ("K", _I64),
                ("grid", ctypes.c_int32), ("y_dtype", ctypes.c_int32)]


class TBError(RuntimeError):
    pass


_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the shared library (raises if it is missing)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise TBError(f"libtb_b200.so not built at {path}; run `python -m decode_gemv_tb_b200.build`")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _lib = lib
    return _lib


def _check(rc: int, what: str):
    if rc != 0:
        msg = load().tb_status_string(rc).decode()
        raise TBError(f"{what}: {STATUS.get(rc, rc)} ({msg})")


def _dev(t: torch.Tensor, name: str) -> int:
    if not t.is_cuda:
        raise TBError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise TBError(f"{name} must be contiguous")
    return t.data_ptr()


def _stream(t: torch.Tensor) -> int:
    return torch.cuda.current_stream(t.device).cuda_stream


def _wdtype(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TBError(f"weights must be float32 or bfloat16, got {t.dtype}")


def _ydtype(dt) -> int:
    if dt == torch.float32:
        return F32
    if dt == torch.bfloat16:
        return BF16
    raise TBError(f"output dtype must be float32 or bfloat16, got {dt}")


def _bits(t: torch.Tensor, name: str) -> int:
    if t.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TBError(f"{name} must hold bf16 bit patterns")
    return _dev(t, name)


# ---- sizes -----------------------------------------------------------------

def wait_timeouts() -> int:
    """Bounded device waits that gave up since the last call (synchronizes)."""
    return int(load().tb_wait_timeouts())


def sync_status(stream: int | None = None) -> int:
    """tb_sync_status on the current stream: 0 (TB_OK), 6 (TB_ERR_TIMEOUT) or 5."""
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    return int(load().tb_sync_status(stream))


def version() -> int:
    return load().tb_version()


def packed_bytes(grid: int, N: int, K: int) -> int:
    return int(load().tb_packed_bytes(grid, N, K))


def scale_bytes(N: int, K: int) -> int:
    return int(load().tb_scale_bytes(N, K))


# ---- entry points -----------------------------------------------------------

def tb_scales_absmax(W: torch.Tensor, grid: int, scales: torch.Tensor | None = None) -> torch.Tensor:
    N, K = W.shape
    if scales is None:
        scales = torch.empty((N, K // 128), dtype=torch.bfloat16, device=W.device)
    _check(load().tb_scales_absmax(_dev(W, "W"), _wdtype(W), N, K, grid, _bits(scales, "scales"), _stream(W)),
           "tb_scales_absmax")
    return scales


def tb_pack(W: torch.Tensor, grid: int, scales: torch.Tensor, packed: torch.Tensor | None = None,
            bad_count: torch.Tensor | None = None) -> torch.Tensor:
    N, K = W.shape
    if packed is None:
        packed = torch.empty(packed_bytes(grid, N, K), dtype=torch.uint8, device=W.device)
    bc = 0 if bad_count is None else _dev(bad_count, "bad_count")
    _check(load().tb_pack(_dev(W, "W"), _wdtype(W), N, K, grid, _bits(scales, "scales"), _dev(packed, "packed"),
                          bc, _stream(W)), "tb_pack")
    return packed


def tb_unpack(packed: torch.Tensor, grid: int, N: int, K: int, codes: torch.Tensor | None = None) -> torch.Tensor:
    if codes is None:
        codes = torch.empty((N, K), dtype=torch.int8, device=packed.device)
    _check(load().tb_unpack(_dev(packed, "packed"), grid, N, K, _dev(codes, "codes"), _stream(packed)), "tb_unpack")
    return codes


def workspace_bytes(M: int, N: int, K: int) -> int:
    return int(load().tb_workspace_bytes(M, N, K))


def workspace(nbytes: int, device) -> torch.Tensor:
    """Caller-owned scratch for the products (256-byte aligned), zero-filled
    once as the batch-1 kernel's counters require (calls leave it zero)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def tb_gemv(packed: torch.Tensor, grid: int, scales: torch.Tensor, x: torch.Tensor, N: int, K: int,
            y: torch.Tensor | None = None, out_dtype=torch.float32, ws: torch.Tensor | None = None) -> torch.Tensor:
    if y is None:
        y = torch.empty(N, dtype=out_dtype, device=x.device)
    if ws is None:
        ws = workspace(workspace_bytes(1, N, K), x.device)
    _check(load().tb_gemv(_dev(packed, "packed"), grid, _bits(scales, "scales"), _bits(x, "x"), _dev(y, "y"),
                          _ydtype(y.dtype), N, K, _dev(ws, "workspace"), ws.numel(), _stream(x)), "tb_gemv")
    return y


def tb_gemv_noalloc(packed: torch.Tensor, grid: int, scales: torch.Tensor, x: torch.Tensor, N: int, K: int,
                    y: torch.Tensor) -> torch.Tensor:
    """tb_gemv over the library's fixed device scratch: no workspace, and
    the caller provides y, so the call itself allocates nothing."""
    _check(load().tb_gemv_noalloc(_dev(packed, "packed"), grid, _bits(scales, "scales"), _bits(x, "x"),
                                  _dev(y, "y"), _ydtype(y.dtype), N, K, _stream(x)), "tb_gemv_noalloc")
    return y


def tb_gemm(packed: torch.Tensor, grid: int, scales: torch.Tensor, X: torch.Tensor, N: int, K: int,
            Y: torch.Tensor | None = None, out_dtype=torch.float32, ws: torch.Tensor | None = None) -> torch.Tensor:
    M = X.shape[0]
    if Y is None:
        Y = torch.empty((M, N), dtype=out_dtype, device=X.device)
    if ws is None:
        ws = workspace(workspace_bytes(M, N, K), X.device)
    _check(load().tb_gemm(_dev(packed, "packed"), grid, _bits(scales, "scales"), _bits(X, "X"), X.stride(0),
                          _dev(Y, "Y"), _ydtype(Y.dtype), Y.stride(0), M, N, K, _dev(ws, "workspace"), ws.numel(),
                          _stream(X)), "tb_gemm")
    return Y


def linear_items(items) -> ctypes.Array:
    """Build a tb_linear_t array from (packed, grid, scales, x, y, N, K)."""
    arr = (Linear * len(items))()
    for i, (packed, grid, scales, x, y, N, K) in enumerate(items):
        arr[i] = Linear(_dev(packed, "packed"), _bits(scales, "scales"), _bits(x, "x"), _dev(y, "y"), N, K, grid,
                        _ydtype(y.dtype))
    return arr


def layer_workspace_bytes(arr: ctypes.Array) -> int:
    return int(load().tb_layer_workspace_bytes(ctypes.cast(arr, ctypes.c_void_p), len(arr)))


def tb_layer_gemv(items, ws: torch.Tensor | None = None, flags: int = 0, stream: int | None = None) -> None:
    """items: list of (packed, grid, scales, x, y, N, K), or a prebuilt
    linear_items() array (reused without re-marshalling)."""
    arr = items if isinstance(items, ctypes.Array) else linear_items(items)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    if ws is None:
        ws = workspace(layer_workspace_bytes(arr), torch.device("cuda", torch.cuda.current_device()))
    _check(load().tb_layer_gemv(ctypes.cast(arr, ctypes.c_void_p), len(arr), flags, ws.data_ptr(), ws.numel(),
                                stream), "tb_layer_gemv")


def gate_up_workspace_bytes(gate, up) -> int:
    """Workspace bytes of tb_gate_up_silu for gate, up: (packed, grid, scales, x, y, N, K)."""
    arr = linear_items([gate, up])
    return int(load().tb_gate_up_workspace_bytes(ctypes.cast(ctypes.byref(arr, 0), ctypes.c_void_p),
                                                  ctypes.cast(ctypes.byref(arr, ctypes.sizeof(Linear)), ctypes.c_void_p)))


def tb_gate_up_silu(gate, up, h: torch.Tensor, ws: torch.Tensor | None = None, flags: int = 0,
                    stream: int | None = None) -> torch.Tensor:
    """gate, up: (packed, grid, scales, x, y, N, K) of equal N and K; writes
    their y and h = bf16(silu(gate) * up) ([N] bf16)."""
    arr = linear_items([gate, up])
    if h.dtype not in (torch.bfloat16, torch.int16, torch.uint16):
        raise TBError("h must hold bf16")
    g_ptr = ctypes.cast(ctypes.byref(arr, 0), ctypes.c_void_p)
    u_ptr = ctypes.cast(ctypes.byref(arr, ctypes.sizeof(Linear)), ctypes.c_void_p)
    if stream is None:
        stream = torch.cuda.current_stream().cuda_stream
    if ws is None:
        ws = workspace(load().tb_gate_up_workspace_bytes(g_ptr, u_ptr), torch.device("cuda", torch.cuda.current_device()))
    _check(load().tb_gate_up_silu(g_ptr, u_ptr, _dev(h, "h"), flags, ws.data_ptr(), ws.numel(), stream),
           "tb_gate_up_silu")
    return h
