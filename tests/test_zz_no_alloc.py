"""tb_gemv_noalloc: tb_gemv over the library's fixed device scratch.

Collected last on purpose, so that it runs both after every other test and,
when selected alone, in a fresh process.  The GPU case calls the entry point
twice in a row, both times on the kernel that uses the scratch (products
above 2^24 weights): a 3-bit gate projection, then a 2-bit problem with a
different tile count and K split, whose K/128 = 36 also makes the call
stage padded scales in the scratch; the second call reuses the scratch
without any clearing in between.  Each output is compared with tb_gemv's
on the same inputs and with the oracle, within the GEMV tolerance
|dy| <= 1e-5 sum_k |x_k w_k| (+ 4e-3 |y| for bf16 outputs)."""
import os
import re

import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth
from decode_gemv_tb_b200 import tb
from tests.helpers import assert_within, u16, w_np

HEADER = os.path.join(os.path.dirname(__file__), "..", "include", "tb.h")
FAKE = 1 << 40  # a 256-byte-aligned address that is never dereferenced
TB_ERR_ARG, TB_ERR_ALIGN, TB_ERR_UNSUPPORTED = 1, 3, 4
ROW_KERNEL_MAX_WEIGHTS = 1 << 24  # tb_gemv runs the row kernel (no scratch) up to this many weights


def needs_scratch(N, K):
    return tb.workspace_bytes(1, N, K)


def test_scratch_size_matches_header():
    src = open(HEADER).read()
    m = re.search(r"#define\s+TB_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert m, "TB_NOALLOC_SCRATCH_BYTES not found in the header"
    assert int(m.group(1)) << int(m.group(2)) == tb.NOALLOC_SCRATCH_BYTES


def test_rejections_before_any_cuda_call():
    """Argument errors and oversized problems are refused on the host (this
    runs without a GPU: no CUDA call is reached)."""
    lib = tb.load()
    f = lib.tb_gemv_noalloc
    # the envelope the header states fits (the scratch does not grow with N); a far larger K does not
    for N in (1 << 12, 1 << 22, 1 << 27):
        assert needs_scratch(N, 1 << 17) <= tb.NOALLOC_SCRATCH_BYTES
    K_big = 1 << 22
    assert needs_scratch(4096, K_big) > tb.NOALLOC_SCRATCH_BYTES
    assert f(FAKE, tb.INT2, FAKE, FAKE, FAKE, tb.F32, 4096, K_big, None) == TB_ERR_UNSUPPORTED
    assert f(FAKE, tb.INT3, FAKE, FAKE, FAKE, tb.BF16, 4096, K_big, None) == TB_ERR_UNSUPPORTED
    assert f(None, tb.INT2, FAKE, FAKE, FAKE, tb.F32, 64, 128, None) == TB_ERR_ARG
    assert f(FAKE, tb.INT2, FAKE, None, FAKE, tb.F32, 64, 128, None) == TB_ERR_ARG
    assert f(FAKE, 9, FAKE, FAKE, FAKE, tb.F32, 64, 128, None) == TB_ERR_ARG
    assert f(FAKE, tb.INT2, FAKE, FAKE + 8, FAKE, tb.F32, 64, 128, None) == TB_ERR_ALIGN
    msg = lib.tb_status_string(TB_ERR_UNSUPPORTED)
    assert msg


@pytest.mark.gpu
def test_two_calls_in_a_row_match_tb_gemv(oracle):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = "cuda:0"
    # a gate projection of an 8B decoder layer (3-bit, fp32 out), then a
    # 2-bit problem (bf16 out) with 16 tiles instead of 48 that reuses the same scratch
    cases = [(tb.INT3, 12288, 4096, torch.float32, 11), (tb.INT2, 4096, 4608, torch.bfloat16, 12)]
    prepared = []
    for grid, N, K, odt, seed in cases:
        assert needs_scratch(N, K) <= tb.NOALLOC_SCRATCH_BYTES
        assert N * K > ROW_KERNEL_MAX_WEIGHTS  # the scratch-using kernel, not the row kernel
        W = synth.gaussian_weights(N, K, seed=seed)
        x = synth.activations(K, seed=seed)
        s_ref = oracle.scales_absmax(w_np(W), grid)
        p_ref, _ = oracle.pack(w_np(W), grid, s_ref)
        y64, yabs = oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K)
        Wd = W.to(dev)
        s = tb.tb_scales_absmax(Wd, grid)
        p = tb.tb_pack(Wd, grid, s)
        prepared.append((grid, N, K, odt, p, s, x.to(dev), y64, yabs))

    outs = []
    for grid, N, K, odt, p, s, x, _, _ in prepared:  # back to back, same stream, no sync in between
        y = torch.full((N,), 7.5, dtype=odt, device=dev)
        tb.tb_gemv_noalloc(p, grid, s, x, N, K, y)
        outs.append(y)
    torch.cuda.synchronize()

    for (grid, N, K, odt, p, s, x, y64, yabs), y in zip(prepared, outs):
        out = "f32" if odt == torch.float32 else "bf16"
        ref = tb.tb_gemv(p, grid, s, x, N, K, out_dtype=odt)
        got = y.float().cpu().numpy().astype(np.float64)
        want = ref.float().cpu().numpy().astype(np.float64)
        tol = oracle.tolerance(oracle.round_out(y64, out), yabs, out)
        assert np.all(np.abs(got - want) <= tol), f"noalloc vs tb_gemv, grid {grid} {N}x{K}"
        assert_within(y, y64, yabs, out, oracle, f"noalloc grid {grid} {N}x{K}")
