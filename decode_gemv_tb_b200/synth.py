"""Seeded synthetic workloads: shapes, per-matrix grid assignments and
random draws.

This module holds random numbers and workload structure only: no
quantization, packing or product arithmetic.  Both the CPU oracle's callers
and the GPU path's callers take their inputs from here, so the two sides
see the same tensors.

The shapes follow the model sizes the ThinkBit page reports results for
(page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로 검증한다",
onedev.kr/papers/1416, sections 무엇과 다른가 and 전제와 한계: Qwen3-1.7B,
8B and 14B); the per-matrix grids reproduce the ratio that page's
allocator reaches on Qwen3-1.7B at a 2.0-bit budget (75.3% ternary, 6.0%
2-bit, 18.7% 3-bit by parameter count, query and key projections at 2 bits
or more).  The checkpoints themselves are not available, so every tensor
here is a seeded random stand-in with the stated distribution.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

TERNARY, INT2, INT3 = 0, 1, 2
GRID_NAMES = {TERNARY: "ternary", INT2: "int2", INT3: "int3"}
GRID_BITS = {TERNARY: 2, INT2: 2, INT3: 3}

PROJ = ("q", "k", "v", "o", "gate", "up", "down")


@dataclass(frozen=True)
class Matrix:
    name: str
    N: int  # output rows
    K: int  # input columns
    grid: int
    seed: int


def qwen3_layer_shapes(hidden: int, mlp: int, kv_dim: int = 1024):
    """(name, N, K) of one decoder layer's seven projections, W = [out][in]."""
    return [
        ("q", hidden, hidden),
        ("k", kv_dim, hidden),
        ("v", kv_dim, hidden),
        ("o", hidden, hidden),
        ("gate", mlp, hidden),
        ("up", mlp, hidden),
        ("down", hidden, mlp),
    ]


# --- config 1: one small 2-bit GEMV -----------------------------------------
CONFIG1 = dict(N=256, K=1024, grid=INT2, seed=1000)

# --- config 2: Qwen3-1.7B-like shapes over all three grids ------------------
CONFIG2_SHAPES = [(2048, 2048), (6144, 2048), (2048, 6144)]
CONFIG2_GRIDS = [TERNARY, INT2, INT3]


def config2_cases():
    out = []
    for si, (N, K) in enumerate(CONFIG2_SHAPES):
        for grid in CONFIG2_GRIDS:
            out.append(Matrix(f"{N}x{K}-{GRID_NAMES[grid]}", N, K, grid, 2000 + 10 * si + grid))
    return out


# --- config 3: Qwen3-8B-like decoder stack (36 layers) ----------------------
CONFIG3_HIDDEN, CONFIG3_MLP, CONFIG3_LAYERS = 4096, 12288, 36
# --- config 4/5: Qwen3-14B-like shapes --------------------------------------
CONFIG4_HIDDEN, CONFIG4_MLP = 5120, 17408
CONFIG4_M = (1, 4, 16, 32, 64)
CONFIG4_GRIDS = (INT2, INT3)
CONFIG5_LAYERS = 40


def mixed_grid_stack(layers: int, o_int2_layers: int, mlp_int3: int, hidden: int, mlp: int, base_seed: int):
    """Per-matrix grids of a decoder stack: every q at 3 bits, every k and v
    at 2 bits, o at 2 bits in the first `o_int2_layers` layers and ternary
    after, `mlp_int3` MLP matrices at 3 bits picked round-robin (gate of
    layer 0, up of layer 1, down of layer 2, gate of layer 3, ...), every
    other MLP matrix ternary."""
    stack = []
    for layer in range(layers):
        mats = []
        for pi, (name, N, K) in enumerate(qwen3_layer_shapes(hidden, mlp)):
            if name == "q":
                grid = INT3
            elif name in ("k", "v"):
                grid = INT2
            elif name == "o":
                grid = INT2 if layer < o_int2_layers else TERNARY
            else:
                mlp_idx = ("gate", "up", "down").index(name)
                grid = INT3 if (layer < mlp_int3 and layer % 3 == mlp_idx) else TERNARY
            mats.append(Matrix(f"L{layer}.{name}", N, K, grid, (base_seed + layer) * 16 + pi))
        stack.append(mats)
    return stack


def config3_stack():
    """36 Qwen3-8B-like layers: 18.84% 3-bit, 6.04% 2-bit, 75.12% ternary."""
    return mixed_grid_stack(CONFIG3_LAYERS, 7, 14, CONFIG3_HIDDEN, CONFIG3_MLP, 3000)


def isolated_layer():
    """One Qwen3-8B-like layer timed on its own: q and o at 3 bits, k and v
    at 2 bits, the MLP ternary."""
    grids = {"q": INT3, "k": INT2, "v": INT2, "o": INT3, "gate": TERNARY, "up": TERNARY, "down": TERNARY}
    return [Matrix(f"iso.{name}", N, K, grids[name], 3900 * 16 + pi)
            for pi, (name, N, K) in enumerate(qwen3_layer_shapes(CONFIG3_HIDDEN, CONFIG3_MLP))]


def config5_stack():
    """40 Qwen3-14B-like layers: 18.73% 3-bit, 5.95% 2-bit, 75.32% ternary."""
    return mixed_grid_stack(CONFIG5_LAYERS, 14, 16, CONFIG4_HIDDEN, CONFIG4_MLP, 5000)


def grid_fractions(stack):
    tot = {TERNARY: 0, INT2: 0, INT3: 0}
    for mats in stack:
        for m in mats:
            tot[m.grid] += m.N * m.K
    s = sum(tot.values())
    return {g: v / s for g, v in tot.items()}


# --- random draws -------------------------------------------------------------

def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def activations(K: int, seed: int, device="cpu", M: int | None = None) -> torch.Tensor:
    """bf16 x ~ N(0, 1): shape [K], or [M][K] when M is given."""
    shape = (K,) if M is None else (M, K)
    return torch.randn(shape, generator=_gen(seed + 7, device), device=device).to(torch.bfloat16)


def outlier_activations(K: int, seed: int, magnitudes=(2.0 ** 10, 2.0 ** 12, 2.0 ** 14), device="cpu",
                        M: int | None = None) -> torch.Tensor:
    """bf16 x ~ N(0, 1) with one outlier channel per 128-group: a position
    drawn uniformly inside the group, set to +-m with m drawn from
    `magnitudes` and a random sign (the few very large activation channels
    of decoder layers).  Shape [K], or [M][K] when M is given (the outlier
    channels are shared by the rows, as a channel is)."""
    g = _gen(seed + 11, device)
    shape = (K,) if M is None else (M, K)
    x = torch.randn(shape, generator=g, device=device)
    G = K // 128
    pos = torch.randint(0, 128, (G,), generator=g, device=device) + 128 * torch.arange(G, device=device)
    mag = torch.tensor(magnitudes, dtype=torch.float32, device=device)[
        torch.randint(0, len(magnitudes), (G,), generator=g, device=device)]
    sign = torch.randint(0, 2, (G,), generator=g, device=device).float() * 2 - 1
    if M is None:
        x[pos] = mag * sign
    else:
        x[:, pos] = (mag * sign).unsqueeze(0) * (1 + torch.rand((M, G), generator=g, device=device))
    return x.to(torch.bfloat16)


def gaussian_weights(N: int, K: int, seed: int, std: float = 0.02, device="cpu", dtype=torch.float32):
    """W ~ N(0, std^2), [N][K], returned in `dtype` (fp32 or bf16)."""
    w = torch.randn((N, K), generator=_gen(seed, device), device=device, dtype=torch.float32)
    return (w * std).to(dtype)


def outlier_weights(N: int, K: int, seed: int, std: float = 0.02, frac: float = 0.001, boost: float = 20.0,
                    device="cpu"):
    """bf16 W ~ N(0, std^2) with round(frac*N*K) entries, chosen uniformly
    without replacement, multiplied by `boost` (heavy-tailed outliers)."""
    g = _gen(seed, device)
    w = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * std
    n_out = int(round(frac * N * K))
    if n_out:
        idx = torch.randperm(N * K, generator=g, device=device)[:n_out]
        w.view(-1)[idx] *= boost
    return w.to(torch.bfloat16)


def uniform_codes(N: int, K: int, lo: int, hi: int, seed: int, device="cpu") -> torch.Tensor:
    """int8 codewords uniform on {lo, ..., hi}."""
    return torch.randint(lo, hi + 1, (N, K), generator=_gen(seed, device), device=device, dtype=torch.int8)


def config1_scales(N: int, K: int, seed: int, device="cpu") -> torch.Tensor:
    """bf16 scales [N][K/128] = |N(0,1)| * 0.02 + 1e-3."""
    s = torch.randn((N, K // 128), generator=_gen(seed + 3, device), device=device).abs() * 0.02 + 1e-3
    return s.to(torch.bfloat16)
