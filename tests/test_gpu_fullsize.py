"""Full-size parity of what the benchmark times: the decoder-layer launches of
the Qwen3-8B-like stack (hidden 4096, MLP 12288) and of the Qwen3-14B-like
stack with outlier weights (hidden 5120, MLP 17408), each one
tb_layer_gemv over the layer's seven projections exactly as bench.py calls
it, and the 14B gate projection at every batch size the benchmark sweeps.

The oracle computes sampled rows one by one (every item's first and last
rows, the rows on both sides of every 256-row tile edge, and random rows):
too slow for every row at these sizes, exact for the rows it does.  The
packs are compared byte for byte in full.  Weights and activations come
from the seeded generators on the CPU; the GPU path quantizes and packs
them itself, as the benchmark does."""
import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth
from decode_gemv_tb_b200 import tb
from tests.helpers import assert_within, u16, u32

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TILE = 256  # rows of the batch-1 kernel's tile


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tb.load()


def sample_rows(N, seed, extra=64):
    rng = np.random.default_rng(seed)
    edges = []
    for e in range(0, N + 1, TILE):
        edges += [e - 2, e - 1, e, e + 1]
    rows = np.concatenate([[0, 1, N - 2, N - 1], edges, rng.integers(0, N, extra)])
    return np.unique(rows[(rows >= 0) & (rows < N)])


def run_layer(oracle, mats, weights, what):
    """One tb_layer_gemv over the layer's matrices; pack bit-exactness in full
    and sampled rows against the oracle."""
    items, refs = [], []
    for m in mats:
        W = weights(m)
        wb = u16(W)
        s_ref = oracle.scales_absmax(wb, m.grid)
        p_ref, _ = oracle.pack(wb, m.grid, s_ref)
        Wd = W.to(DEV)
        s = tb.tb_scales_absmax(Wd, m.grid)
        p = tb.tb_pack(Wd, m.grid, s)
        del Wd
        assert np.array_equal(u16(s), s_ref), f"{what} {m.name}: scales"
        assert np.array_equal(u32(p).reshape(p_ref.shape), p_ref), f"{what} {m.name}: pack"
        x = synth.activations(m.K, seed=m.seed)
        rows = sample_rows(m.N, m.seed)
        refs.append((rows, oracle.gemv_rows64(p_ref, m.grid, s_ref, u16(x), m.K, rows)))
        items.append((p, m.grid, s, x.to(DEV), torch.full((m.N,), 7.0, dtype=torch.float32, device=DEV), m.N, m.K))
    arr = tb.linear_items(items)
    ws = tb.workspace(tb.layer_workspace_bytes(arr), DEV)
    tb.tb_layer_gemv(arr, ws, 0)
    assert tb.sync_status() == 0
    first = [it[4].clone() for it in items]
    tb.tb_layer_gemv(arr, ws, 0)
    assert tb.sync_status() == 0
    for m, it, (rows, (y64, yabs)), y1 in zip(mats, items, refs, first):
        y = it[4].cpu()
        assert_within(y[rows], y64, yabs, "f32", oracle, f"{what} {m.name}")
        assert torch.equal(it[4], y1), f"{what} {m.name}: not deterministic"


def test_config3_layer0(oracle):
    mats = synth.config3_stack()[0]
    run_layer(oracle, mats, lambda m: synth.gaussian_weights(m.N, m.K, seed=m.seed, dtype=torch.bfloat16),
              "8B layer 0")


def test_config3_isolated_layer(oracle):
    mats = synth.isolated_layer()
    run_layer(oracle, mats, lambda m: synth.gaussian_weights(m.N, m.K, seed=m.seed, dtype=torch.bfloat16),
              "8B isolated layer")


@pytest.mark.parametrize("layer", [0, 2])
def test_config5_outlier_layers(oracle, layer):
    """Layer 0 (q and gate at 3 bits) and layer 2 (q and down at 3 bits) of
    the 40-layer 14B-like stack, outlier weights (0.1% of entries x20)."""
    mats = synth.config5_stack()[layer]
    run_layer(oracle, mats, lambda m: synth.outlier_weights(m.N, m.K, seed=m.seed), f"14B layer {layer}")


@pytest.mark.parametrize("grid", [tb.INT2, tb.INT3])
@pytest.mark.parametrize("M", [1, 4, 16, 32, 64])
def test_config4_gate_every_batch(oracle, grid, M):
    """The 14B gate projection (17408 x 5120) at each batch size of the
    benchmark's sweep, through tb_gemm as the benchmark calls it."""
    N, K = synth.CONFIG4_MLP, synth.CONFIG4_HIDDEN
    W = synth.gaussian_weights(N, K, seed=4000 + grid)
    s_ref = oracle.scales_absmax(W.numpy(), grid)
    p_ref, _ = oracle.pack(W.numpy(), grid, s_ref)
    p = torch.from_numpy(p_ref.reshape(-1).view(np.uint8).copy()).to(DEV)
    s = torch.from_numpy(s_ref.view(np.int16).copy()).to(DEV).view(torch.bfloat16)
    X = synth.outlier_activations(K, seed=4100 + M, M=M)
    Y = tb.tb_gemm(p, grid, s, X.to(DEV), N, K)
    assert tb.sync_status() == 0
    Y = Y.cpu()
    Xb = u16(X)
    rows = sample_rows(N, M + 10 * grid, extra=48)
    for m in range(M):
        y64, yabs = oracle.gemv_rows64(p_ref, grid, s_ref, Xb[m], K, rows)
        assert_within(Y[m, rows], y64, yabs, "f32", oracle, f"gate M={M} m={m}")
