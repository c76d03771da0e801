"""Python face of the CPU oracle (``tb_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The library never
imports this module, and this module imports nothing from the library.

All arithmetic of the method lives in the C file (plain loops, fp64); this
wrapper only moves numpy arrays across ctypes and performs the final
fp64 -> fp32 (-> bf16) output roundings, which numpy and the C helper do
round-half-to-even.

Source of the method: ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력
보존을 추론 평가로 검증한다" (onedev.kr/papers/1416), section 어떻게 동작하나
("how it works"): w = c * s, integer codeword c on a per-layer grid, one
bf16 scale per 128 weights, dequantization is one multiply.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tb_oracle.c")
LIB = os.path.join(HERE, "libtb_oracle.so")

TERNARY, INT2, INT3 = 0, 1, 2
GRIDS = (TERNARY, INT2, INT3)
# the ternary grid in the optional 5-trits-per-byte layout
TERNARY_B3 = 3
GRID_NAMES = {TERNARY: "ternary", INT2: "int2", INT3: "int3", TERNARY_B3: "ternary_b3"}
# [how it works]: the three codeword grids
GRID_RANGE = {TERNARY: (-1, 1), INT2: (-2, 1), INT3: (-4, 3), TERNARY_B3: (-1, 1)}
GROUP = 128

CFLAGS = ["-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c11", "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        cmd = ["gcc", *CFLAGS, "-o", LIB, SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        I64 = ctypes.c_int64
        L.tbo_bf16_round.argtypes = [ctypes.c_float]
        L.tbo_bf16_round.restype = ctypes.c_uint16
        L.tbo_bf16_to_double.argtypes = [ctypes.c_uint16]
        L.tbo_bf16_to_double.restype = ctypes.c_double
        L.tbo_quantize.argtypes = [ctypes.c_float, ctypes.c_uint16, ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
        L.tbo_quantize.restype = ctypes.c_int
        L.tbo_scales_absmax.argtypes = [P, I64, I64, ctypes.c_int, P]
        L.tbo_pack.argtypes = [P, I64, I64, ctypes.c_int, P, P, ctypes.POINTER(I64)]
        L.tbo_unpack.argtypes = [P, ctypes.c_int, I64, I64, P]
        L.tbo_gemv.argtypes = [P, ctypes.c_int, P, P, I64, I64, P, P]
        L.tbo_gemm.argtypes = [P, ctypes.c_int, P, P, I64, I64, I64, I64, P, P]
        L.tbo_gemv_rows.argtypes = [P, ctypes.c_int, P, P, I64, P, I64, P, P]
        L.tbo_silu.argtypes = [ctypes.c_double]
        L.tbo_silu.restype = ctypes.c_double
        L.tbo_swiglu.argtypes = [P, P, I64, P]
        L.tbo_swiglu.restype = ctypes.c_int
        L.tbo_row_words.argtypes = [ctypes.c_int, I64]
        L.tbo_row_words.restype = I64
        for f in ("tbo_scales_absmax", "tbo_pack", "tbo_unpack", "tbo_gemv", "tbo_gemm", "tbo_gemv_rows"):
            getattr(L, f).restype = ctypes.c_int
        L.tbo_rounding_is_nearest.restype = ctypes.c_int
        assert L.tbo_rounding_is_nearest() == 1
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what}: bad arguments")


# ---- bf16 helpers (uint16 bit patterns) ------------------------------------

def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp32."""
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (half to even) with the oracle's scalar rule."""
    f = np.ascontiguousarray(f, dtype=np.float32)
    L = lib()
    out = np.empty(f.shape, dtype=np.uint16)
    fo, oo = f.reshape(-1), out.reshape(-1)
    for i in range(fo.size):
        oo[i] = L.tbo_bf16_round(float(fo[i]))
    return out


def _as_w32(W: np.ndarray) -> np.ndarray:
    """Accept fp32 weights, or bf16 weights given as uint16 bit patterns."""
    if W.dtype == np.uint16:
        return bf16_bits_to_f32(W)
    return np.ascontiguousarray(W, dtype=np.float32)


# ---- the method ------------------------------------------------------------

def row_words(grid: int, K: int) -> int:
    return int(lib().tbo_row_words(grid, K))


def packed_bytes(grid: int, N: int, K: int) -> int:
    return 4 * N * row_words(grid, K)


def quantize(w: float, scale_bits: int, grid: int):
    bad = ctypes.c_int(0)
    c = lib().tbo_quantize(float(w), int(scale_bits), grid, ctypes.byref(bad))
    return int(c), int(bad.value)


def scales_absmax(W: np.ndarray, grid: int) -> np.ndarray:
    W32 = _as_w32(W)
    N, K = W32.shape
    out = np.empty((N, K // GROUP), dtype=np.uint16)
    _check(lib().tbo_scales_absmax(_ptr(W32), N, K, grid, _ptr(out)), "scales_absmax")
    return out


def pack(W: np.ndarray, grid: int, scales: np.ndarray):
    """Return (packed uint32 [N][row_words], count of R3 weights)."""
    W32 = _as_w32(W)
    N, K = W32.shape
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    out = np.empty((N, row_words(grid, K)), dtype=np.uint32)
    bad = ctypes.c_int64(0)
    _check(lib().tbo_pack(_ptr(W32), N, K, grid, _ptr(scales), _ptr(out), ctypes.byref(bad)), "pack")
    return out, int(bad.value)


def unpack(packed: np.ndarray, grid: int, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint32).reshape(N, row_words(grid, K))
    out = np.empty((N, K), dtype=np.int8)
    _check(lib().tbo_unpack(_ptr(packed), grid, N, K, _ptr(out)), "unpack")
    return out


def gemv64(packed, grid, scales, x_bits, N, K):
    """fp64 y[N] and the bound scale sum_k |x_k w_k| [N]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    y = np.empty(N, dtype=np.float64)
    yabs = np.empty(N, dtype=np.float64)
    _check(lib().tbo_gemv(_ptr(packed), grid, _ptr(scales), _ptr(x_bits), N, K, _ptr(y), _ptr(yabs)), "gemv")
    return y, yabs


def gemv_rows64(packed, grid, scales, x_bits, K, rows):
    """fp64 outputs of the listed rows only (for sampled checks)."""
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    y = np.empty(rows.size, dtype=np.float64)
    yabs = np.empty(rows.size, dtype=np.float64)
    _check(lib().tbo_gemv_rows(_ptr(packed), grid, _ptr(scales), _ptr(x_bits), K, _ptr(rows), rows.size,
                               _ptr(y), _ptr(yabs)), "gemv_rows")
    return y, yabs


def gemm64(packed, grid, scales, X_bits, N, K):
    """fp64 Y[M][N] (= X W^T) and the bound scales [M][N]."""
    packed = np.ascontiguousarray(packed, dtype=np.uint32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    M = X_bits.shape[0]
    Y = np.empty((M, N), dtype=np.float64)
    Yabs = np.empty((M, N), dtype=np.float64)
    _check(lib().tbo_gemm(_ptr(packed), grid, _ptr(scales), _ptr(X_bits), K, M, N, K, _ptr(Y), _ptr(Yabs)), "gemm")
    return Y, Yabs


def silu(g: float) -> float:
    """silu(g) = g / (1 + e^-g) in fp64 (reading R9)."""
    return float(lib().tbo_silu(float(g)))


def swiglu64(g64: np.ndarray, u64: np.ndarray) -> np.ndarray:
    """h = silu(g) * u elementwise in fp64 (the down projection's input)."""
    g64 = np.ascontiguousarray(g64, dtype=np.float64)
    u64 = np.ascontiguousarray(u64, dtype=np.float64)
    assert g64.shape == u64.shape
    h = np.empty_like(g64)
    _check(lib().tbo_swiglu(_ptr(g64), _ptr(u64), g64.size, _ptr(h)), "swiglu")
    return h


def round_out(y64: np.ndarray, out_dtype: str) -> np.ndarray:
    """Output rounding (reading R8): fp64 -> fp32 RNE; bf16 = RNE of that
    fp32, returned widened to fp32 for comparison."""
    y32 = np.asarray(y64, dtype=np.float64).astype(np.float32)
    if out_dtype == "f32":
        return y32
    if out_dtype == "bf16":
        return bf16_bits_to_f32(f32_to_bf16_bits(y32))
    raise ValueError(out_dtype)


def tolerance(y_ref32: np.ndarray, yabs: np.ndarray, out_dtype: str) -> np.ndarray:
    """Allowed |y - y_ref|: 1e-5 * sum|x w| for fp32 outputs, plus
    4e-3 * |y_ref| for bf16 outputs."""
    tol = 1e-5 * np.asarray(yabs, dtype=np.float64)
    if out_dtype == "bf16":
        tol = tol + 4e-3 * np.abs(np.asarray(y_ref32, dtype=np.float64))
    return tol


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
