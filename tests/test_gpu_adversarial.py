"""Inputs aimed at the arithmetic of the products rather than at their
shapes: rows and 128-groups whose codes are all zero, and activations with
one very large channel per group (2^10 .. 2^14, as the few outlier
channels of decoder layers are) that mostly meets zero codes under
round-to-nearest ternary, 2-bit and 3-bit quantization.

The bound |y - y_ref| <= 1e-5 sum_k |x_k c_k s_k| counts only nonzero
codes (ThinkBit page, section 어떻게 동작하나: w = c * s, so a zero codeword
contributes nothing).  An all-zero row therefore has tolerance exactly 0,
and an outlier that meets a zero code must leave no trace in y.  Every
product path is exercised: the row kernel and the stream-K kernel at batch
1 (one-item and seven-item grouped launches), the small-batch kernel
(2 <= M < 32) and the tensor-core kernel (M >= 32)."""
import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth
from decode_gemv_tb_b200 import tb
from tests.helpers import assert_within, u16, w_np

pytestmark = pytest.mark.gpu
GRIDS = (tb.TERNARY, tb.INT2, tb.INT3)
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tb.load()


def to_dev_packed(p_ref):
    return torch.from_numpy(p_ref.reshape(-1).view(np.uint8).copy()).to(DEV)


def to_dev_bits(a):
    return torch.from_numpy(a.astype(np.uint16).view(np.int16).copy()).to(DEV).view(torch.bfloat16)


ZERO_ROWS = (0, 5, 131, 255, 256)


def zeroed_weights(N, K, seed):
    """N(0, 0.02) weights with whole zero rows and a few zero groups."""
    W = synth.gaussian_weights(N, K, seed=seed)
    for n in ZERO_ROWS:
        if n < N:
            W[n] = 0.0
    W[7, 0:128] = 0.0
    W[8, 128:256] = 0.0
    W[N - 1, K - 128:K] = 0.0
    return W


def problem(oracle, grid, N, K, seed, zero=True):
    W = zeroed_weights(N, K, seed) if zero else synth.gaussian_weights(N, K, seed=seed)
    s_ref = oracle.scales_absmax(w_np(W), grid)
    p_ref, _ = oracle.pack(w_np(W), grid, s_ref)
    return p_ref, s_ref


def check(y, y64, yabs, out, oracle, what, zero_rows):
    assert_within(y, y64, yabs, out, oracle, what)
    got = y.float().cpu().numpy()
    for n in zero_rows:
        if n < got.shape[-1]:
            assert np.all(got[..., n] == 0.0), f"{what}: all-zero row {n} gave {got[..., n]}"


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("api", ["gemv_row", "gemv_streamk", "layer1"])
def test_batch1_zero_rows_and_outliers(oracle, grid, api):
    N, K = 300, 2048
    p_ref, s_ref = problem(oracle, grid, N, K, seed=8100 + grid)
    x = synth.outlier_activations(K, seed=8200 + grid)
    y64, yabs = oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K)
    p, s, xd = to_dev_packed(p_ref), to_dev_bits(s_ref), x.to(DEV)
    y = torch.full((N,), 7.0, dtype=torch.float32, device=DEV)
    if api == "gemv_row":  # below 2^24 weights tb_gemv runs the row kernel
        tb.tb_gemv(p, grid, s, xd, N, K, y=y)
    else:  # the stream-K kernel, through the grouped launcher
        tb.tb_layer_gemv([(p, grid, s, xd, y, N, K)])
    torch.cuda.synchronize()
    check(y, y64, yabs, "f32", oracle, f"{api} grid {grid}", ZERO_ROWS)


@pytest.mark.parametrize("mag", [2.0 ** 10, 2.0 ** 12, 2.0 ** 14])
def test_layer_seven_items_outliers(oracle, mag):
    """A reduced-width decoder layer in one grouped launch, every item with
    zero rows and outlier activations of one magnitude."""
    shapes = synth.qwen3_layer_shapes(512, 1536, kv_dim=384)
    grids = [tb.INT3, tb.INT2, tb.INT2, tb.TERNARY, tb.INT3, tb.TERNARY, tb.TERNARY]
    items, refs = [], []
    for i, ((name, N, K), grid) in enumerate(zip(shapes, grids)):
        p_ref, s_ref = problem(oracle, grid, N, K, seed=8300 + i)
        x = synth.outlier_activations(K, seed=8400 + i, magnitudes=(mag,))
        refs.append(oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K))
        items.append((to_dev_packed(p_ref), grid, to_dev_bits(s_ref), x.to(DEV),
                      torch.full((N,), 7.0, dtype=torch.float32, device=DEV), N, K))
    tb.tb_layer_gemv(items)
    torch.cuda.synchronize()
    for i, it in enumerate(items):
        check(it[4], *refs[i], "f32", oracle, f"{shapes[i][0]} 2^{int(np.log2(mag))}", ZERO_ROWS)


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("M", [2, 4, 16, 31, 32, 48, 64])
def test_gemm_zero_rows_and_outliers(oracle, grid, M):
    N, K = 300, 1024
    p_ref, s_ref = problem(oracle, grid, N, K, seed=8500 + grid)
    X = synth.outlier_activations(K, seed=8600 + M, M=M)
    Y64, Yabs = oracle.gemm64(p_ref, grid, s_ref, u16(X), N, K)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K)
    torch.cuda.synchronize()
    check(Y, Y64, Yabs, "f32", oracle, f"gemm M={M} grid {grid}", ZERO_ROWS)


@pytest.mark.parametrize("grid", GRIDS)
def test_all_zero_matrix(oracle, grid):
    """Every code zero: y must be exactly zero on every path, whatever x."""
    N, K = 264, 1024
    W = torch.zeros(N, K)
    s_ref = oracle.scales_absmax(w_np(W), grid)
    p_ref, _ = oracle.pack(w_np(W), grid, s_ref)
    p, s = to_dev_packed(p_ref), to_dev_bits(s_ref)
    x = synth.outlier_activations(K, seed=8700)
    outs = [tb.tb_gemv(p, grid, s, x.to(DEV), N, K)]
    y = torch.full((N,), 7.0, dtype=torch.float32, device=DEV)
    tb.tb_layer_gemv([(p, grid, s, x.to(DEV), y, N, K)])
    outs.append(y)
    for M in (4, 32, 64):
        outs.append(tb.tb_gemm(p, grid, s, synth.outlier_activations(K, seed=8800 + M, M=M).to(DEV), N, K))
    torch.cuda.synchronize()
    for o in outs:
        assert torch.all(o == 0), f"grid {grid}: nonzero output from an all-zero matrix"


def test_zz_no_bounded_wait_gave_up():
    torch.cuda.synchronize()
    assert tb.wait_timeouts() == 0
