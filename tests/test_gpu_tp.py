"""The tensor-parallel shards (decode_gemv_tb_b200/tp.py) through the GPU
product: each rank's shard of a Qwen3-8B-like down projection (row-parallel,
4096 x 12288) and gate projection (column-parallel, 12288 x 4096) is
multiplied by tb_gemv one after the other on this GPU, and the host sums the
row-parallel partials / concatenates the column-parallel rows (what the
all_reduce / all_gather of a multi-GPU run does); the result must be within
the product bound of the oracle's full product, summed partials adding one
fp32 rounding per rank.  No kernel waits on another."""
import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth, tb, tp
from tests.helpers import u16

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tb.load()


@pytest.mark.parametrize("world", [2, 4, 8])
@pytest.mark.parametrize("case", [("row", tb.TERNARY, 4096, 12288), ("column", tb.INT3, 12288, 4096),
                                  ("row", tb.INT2, 4096, 4096)])
def test_shards_assemble_to_the_full_product(oracle, world, case):
    kind, grid, N, K = case
    W = synth.gaussian_weights(N, K, seed=8800 + N + grid)
    s_ref = oracle.scales_absmax(W.numpy(), grid)
    p_ref, _ = oracle.pack(W.numpy(), grid, s_ref)
    x = synth.activations(K, seed=8900 + grid)
    y64, yabs = oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K)
    pt = torch.from_numpy(p_ref.reshape(-1).view(np.uint8).copy()).to(DEV)
    st = torch.from_numpy(s_ref.view(np.int16).copy()).to(DEV).view(torch.bfloat16)
    xd = x.to(DEV)
    parts = []
    for r in range(world):
        if kind == "row":
            p, s, g0, g1 = tp.row_shard(pt, st, grid, N, K, r, world)
            parts.append(tb.tb_gemv(p, grid, s.view(torch.bfloat16), xd[g0 * 128:g1 * 128].contiguous(), N,
                                    (g1 - g0) * 128))
        else:
            p, s, n0, n1 = tp.column_shard(pt, st, grid, N, K, r, world)
            parts.append(tb.tb_gemv(p, grid, s.view(torch.bfloat16), xd, n1 - n0, K))
    assert tb.sync_status() == 0
    if kind == "row":
        y = torch.zeros(N, dtype=torch.float32, device=DEV)
        for part in parts:
            y += part
    else:
        y = torch.cat(parts)
    got = y.cpu().numpy().astype(np.float64)
    tol = 1e-5 * yabs + world * 2.0 ** -24 * yabs
    bad = np.nonzero(~(np.abs(got - y64) <= tol))[0]
    assert bad.size == 0, f"{kind} x{world}: {bad.size} out of tolerance"
