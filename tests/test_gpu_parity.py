"""CUDA path vs the CPU oracle, element by element, through the C
interface.  Pack and unpack must be bit-exact; GEMV / GEMM outputs must be
within |y - y_ref| <= 1e-5 * sum_k |x_k w_k| (fp32) or that plus
4e-3 |y_ref| (bf16).  The oracle always packs from the same weights
itself; nothing it consumes comes from the GPU."""
import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth
from decode_gemv_tb_b200 import tb
from tests.helpers import assert_within, u16, u32, w_np

pytestmark = pytest.mark.gpu
GRIDS = (tb.TERNARY, tb.INT2, tb.INT3)
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tb.load()


def gpu_quantize(W, grid):
    s = tb.tb_scales_absmax(W, grid)
    bad = torch.zeros(1, dtype=torch.int32, device=W.device)
    p = tb.tb_pack(W, grid, s, bad_count=bad)
    return s, p, int(bad.item())


# ------------------------------------------------------------------ pack

@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("wdt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(1, 128), (5, 256), (37, 640), (256, 1024), (2048, 2048)])
def test_scales_pack_unpack_bitexact(oracle, grid, wdt, shape):
    N, K = shape
    W = synth.gaussian_weights(N, K, seed=N * 7 + K + grid, dtype=wdt).to(DEV)
    s, p, bad = gpu_quantize(W, grid)
    ws = w_np(W)
    s_ref = oracle.scales_absmax(ws, grid)
    assert np.array_equal(u16(s), s_ref)
    p_ref, bad_ref = oracle.pack(ws, grid, s_ref)
    assert np.array_equal(u32(p).reshape(p_ref.shape), p_ref)
    assert bad == bad_ref == 0
    codes = tb.tb_unpack(p, grid, N, K)
    assert np.array_equal(codes.cpu().numpy(), oracle.unpack(p_ref, grid, N, K))


def test_config1_exact_reconstruction(oracle):
    """Config 1: codewords uniform on {-2..1}, scales |N(0,1)|*0.02+1e-3,
    W = c*s in fp32; packing with those scales must give back c."""
    N, K = synth.CONFIG1["N"], synth.CONFIG1["K"]
    c = synth.uniform_codes(N, K, -2, 1, seed=1000)
    s = synth.config1_scales(N, K, seed=1000)
    W = (c.float() * s.float().repeat_interleave(128, dim=1)).to(DEV)
    p = tb.tb_pack(W, tb.INT2, s.to(DEV))
    assert np.array_equal(tb.tb_unpack(p, tb.INT2, N, K).cpu().numpy(), c.numpy())
    p_ref, _ = oracle.pack(W.cpu().numpy(), tb.INT2, u16(s))
    assert np.array_equal(u32(p).reshape(p_ref.shape), p_ref)


@pytest.mark.parametrize("grid", GRIDS)
def test_pack_edge_values(oracle, grid):
    """Ties, clamps, NaN/Inf weights, invalid and tiny scales, subnormals."""
    rng = np.random.default_rng(7 + grid)
    N, K = 8, 256
    sv = np.array([1.0, 0.5, 3.0, 0.375, 1e-20, 2.0 ** -126, 0.0, -1.0, np.inf, np.nan, 1e-38, 7.0e-39,
                   0.015625, 1.5e-3, 2.0 ** -135, 4.0], dtype=np.float32)[: N * 2].reshape(N, 2)
    s = torch.from_numpy(sv).to(torch.bfloat16)
    sval = s.float().numpy()
    W = np.empty((N, K), dtype=np.float32)
    for n in range(N):
        for j in range(2):
            base = sval[n, j] if np.isfinite(sval[n, j]) and sval[n, j] > 0 else 1.0
            k2 = rng.integers(-11, 12, size=128)          # odd/even multiples of s/2: ties and exact codes
            blk = (k2 * np.float64(base) / 2).astype(np.float32)
            blk[::7] = np.nextafter(blk[::7], np.float32(np.inf))
            blk[::11] = np.nextafter(blk[::11], np.float32(-np.inf))
            blk[5] = np.nan
            blk[6] = np.inf
            blk[9] = -np.inf
            blk[10] = 3e38
            blk[12] = 1e-45
            W[n, 128 * j:128 * (j + 1)] = blk
    Wt = torch.from_numpy(W).to(DEV)
    bad = torch.zeros(1, dtype=torch.int32, device=DEV)
    p = tb.tb_pack(Wt, grid, s.to(DEV), bad_count=bad)
    p_ref, bad_ref = oracle.pack(W, grid, u16(s))
    assert np.array_equal(u32(p).reshape(p_ref.shape), p_ref)
    assert int(bad.item()) == bad_ref > 0
    # the scales rule on the same data (NaN / Inf ignored, zero groups -> 1.0)
    W2 = W.copy()
    W2[3, :128] = 0.0
    s_gpu = tb.tb_scales_absmax(torch.from_numpy(W2).to(DEV), grid)
    assert np.array_equal(u16(s_gpu), oracle.scales_absmax(W2, grid))


def test_pack_outliers_bf16(oracle):
    """Config 5 distribution: bf16 N(0, 0.02) with 0.1% entries x20."""
    W = synth.outlier_weights(512, 1024, seed=5001).to(DEV)
    for grid in GRIDS:
        s, p, bad = gpu_quantize(W, grid)
        s_ref = oracle.scales_absmax(u16(W), grid)
        p_ref, _ = oracle.pack(u16(W), grid, s_ref)
        assert np.array_equal(u16(s), s_ref)
        assert np.array_equal(u32(p).reshape(p_ref.shape), p_ref)


# ------------------------------------------------------------------ GEMV

def oracle_problem(oracle, grid, N, K, seed, wdt=torch.float32):
    W = synth.gaussian_weights(N, K, seed=seed, dtype=wdt)
    x = synth.activations(K, seed=seed)
    ws = w_np(W)
    s_ref = oracle.scales_absmax(ws, grid)
    p_ref, _ = oracle.pack(ws, grid, s_ref)
    return W, x, s_ref, p_ref


def to_dev_packed(p_ref):
    return torch.from_numpy(p_ref.reshape(-1).view(np.uint8).copy()).to(DEV)


def to_dev_bits(a):
    return torch.from_numpy(a.astype(np.uint16).view(np.int16).copy()).to(DEV).view(torch.bfloat16)


# Batch-1 products go through two kernels: tb_gemv runs the single-launch row
# kernel up to 2^24 weights (the stream-K TMA kernel above), tb_layer_gemv
# always the stream-K kernel.  "layer" runs the same case through a one-item
# tb_layer_gemv.
APIS = ("gemv", "layer")
ROW_PATH_MAX_WEIGHTS = 1 << 24


def gemv_via(api, p, grid, s, x, N, K, y):
    if api == "gemv":
        tb.tb_gemv(p, grid, s, x, N, K, y=y)
    else:
        tb.tb_layer_gemv([(p, grid, s, x, y, N, K)])
    return y


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("shape", [(1, 128), (7, 256), (15, 384), (16, 1152), (17, 640), (33, 1024), (100, 2048),
                                   (256, 1024)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
@pytest.mark.parametrize("api", APIS)
def test_gemv_parity_small(oracle, grid, shape, out, api):
    N, K = shape
    W, x, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=N * 31 + K)
    y64, yabs = oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K)
    # GPU pipeline from the same W: scales, pack, GEMV
    s, p, _ = gpu_quantize(W.to(DEV), grid)
    guard = 64
    ybuf = torch.full((N + guard,), 123.25, dtype=torch.float32 if out == "f32" else torch.bfloat16, device=DEV)
    y = ybuf[:N]
    gemv_via(api, p, grid, s, x.to(DEV), N, K, y)
    assert_within(y, y64, yabs, out, oracle, f"{api} {shape} grid {grid}")
    assert torch.all(ybuf[N:] == 123.25), "wrote past the end of y"


@pytest.mark.parametrize("case", synth.config2_cases(), ids=lambda m: m.name)
@pytest.mark.parametrize("api", APIS)
def test_gemv_config2(oracle, case, api):
    N, K, grid = case.N, case.K, case.grid
    W, x, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=case.seed)
    y64, yabs = oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K)
    y = gemv_via(api, to_dev_packed(p_ref), grid, to_dev_bits(s_ref), x.to(DEV), N, K,
                 torch.empty(N, dtype=torch.float32, device=DEV))
    assert_within(y, y64, yabs, "f32", oracle, f"{case.name} {api}")


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("N", [ROW_PATH_MAX_WEIGHTS // 4096, ROW_PATH_MAX_WEIGHTS // 4096 + 1])
def test_gemv_path_boundary(oracle, grid, N):
    """tb_gemv at exactly 2^24 weights (row kernel) and one row more
    (stream-K kernel)."""
    K = 4096
    W, x, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=3000 + N + grid)
    y64, yabs = oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K)
    y = tb.tb_gemv(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), x.to(DEV), N, K)
    assert_within(y, y64, yabs, "f32", oracle, f"boundary {N}x{K} grid {grid}")


def test_gemv_config1(oracle):
    N, K = synth.CONFIG1["N"], synth.CONFIG1["K"]
    c = synth.uniform_codes(N, K, -2, 1, seed=1000)
    s = synth.config1_scales(N, K, seed=1000)
    W = c.float() * s.float().repeat_interleave(128, dim=1)
    x = synth.activations(K, seed=1000)
    p_ref, _ = oracle.pack(W.numpy(), tb.INT2, u16(s))
    y64, yabs = oracle.gemv64(p_ref, tb.INT2, u16(s), u16(x), N, K)
    p = tb.tb_pack(W.to(DEV), tb.INT2, s.to(DEV))
    y = tb.tb_gemv(p, tb.INT2, s.to(DEV), x.to(DEV), N, K)
    assert_within(y, y64, yabs, "f32", oracle, "config1")


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("api", APIS)
def test_gemv_integer_exact_bitwise(oracle, grid, api):
    """Integer x and power-of-two scales: every partial sum is exact, so the
    GPU result equals the oracle's bit for bit."""
    lo, hi = oracle.GRID_RANGE[grid]
    N, K = 48, 1024
    g = torch.Generator().manual_seed(99 + grid)
    c = torch.randint(lo, hi + 1, (N, K), generator=g)
    x = torch.randint(-8, 9, (K,), generator=g).to(torch.bfloat16)
    s = torch.full((N, K // 128), 2.0 ** -5, dtype=torch.bfloat16)
    W = c.float() * 2.0 ** -5
    p_ref, _ = oracle.pack(W.numpy(), grid, u16(s))
    y64, _ = oracle.gemv64(p_ref, grid, u16(s), u16(x), N, K)
    y = gemv_via(api, to_dev_packed(p_ref), grid, s.to(DEV), x.to(DEV), N, K,
                 torch.empty(N, dtype=torch.float32, device=DEV))
    assert np.array_equal(y.cpu().numpy(), y64.astype(np.float32))


def test_gemv_deterministic():
    N, K = 1024, 4096
    W = synth.gaussian_weights(N, K, seed=5, device=DEV)
    x = synth.activations(K, seed=5, device=DEV)
    for grid in GRIDS:
        s, p, _ = gpu_quantize(W, grid)
        for api in APIS:
            y1 = gemv_via(api, p, grid, s, x, N, K, torch.empty(N, dtype=torch.float32, device=DEV))
            y2 = gemv_via(api, p, grid, s, x, N, K, torch.empty(N, dtype=torch.float32, device=DEV))
            assert torch.equal(y1, y2)


# ------------------------------------------------------------------ grouped layer

def test_layer_gemv_mixed_grids(oracle):
    """Seven projections of reduced width, each on its own grid, one launch:
    within tolerance of the oracle, and the same bits when repeated.  (The
    split of K across warps is chosen per launch, so a grouped launch and a
    lone GEMV of the same matrix may round differently; both are bounded.)"""
    shapes = synth.qwen3_layer_shapes(512, 1536, kv_dim=128)
    grids = [tb.INT3, tb.INT2, tb.INT2, tb.TERNARY, tb.INT3, tb.TERNARY, tb.TERNARY]
    items, refs, singles = [], [], []
    for i, ((name, N, K), grid) in enumerate(zip(shapes, grids)):
        W, x, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=400 + i)
        refs.append(oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K))
        p, s, xd = to_dev_packed(p_ref), to_dev_bits(s_ref), x.to(DEV)
        y = torch.empty(N, dtype=torch.float32 if i % 2 == 0 else torch.bfloat16, device=DEV)
        items.append((p, grid, s, xd, y, N, K))
        singles.append(tb.tb_gemv(p, grid, s, xd, N, K, out_dtype=y.dtype))
    tb.tb_layer_gemv(items)
    first = [it[4].clone() for it in items]
    tb.tb_layer_gemv(items)
    for i, it in enumerate(items):
        y = it[4]
        assert_within(y, *refs[i], "f32" if i % 2 == 0 else "bf16", oracle, shapes[i][0])
        assert_within(singles[i], *refs[i], "f32" if i % 2 == 0 else "bf16", oracle, shapes[i][0])
        assert torch.equal(y, first[i])


# ------------------------------------------------------------------ GEMM

@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("M", [1, 2, 4, 8, 9, 16, 17, 32, 64])
def test_gemm_parity(oracle, grid, M):
    N, K = 80, 768
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=700 + M)
    X = synth.activations(K, seed=800 + M, M=M)
    Y64, Yabs = oracle.gemm64(p_ref, grid, s_ref, u16(X), N, K)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K)
    assert_within(Y, Y64, Yabs, "f32", oracle, f"gemm M={M}")


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("M", [17, 32, 64])
def test_gemm_row_magnitudes(oracle, grid, M):
    """Batch rows 2^-45 .. 2^45 apart.  From M = 32 a group's activations share
    one power-of-two exponent over the batch rows; every row must still be
    within the tolerance of its own exact sum."""
    N, K = 200, 1024
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=1500 + M)
    g = torch.Generator().manual_seed(1600 + M)
    e = torch.randint(-45, 46, (M, 1), generator=g).float()
    X = (torch.randn(M, K, generator=g) * torch.exp2(e)).to(torch.bfloat16)
    Y64, Yabs = oracle.gemm64(p_ref, grid, s_ref, u16(X), N, K)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K)
    assert_within(Y, Y64, Yabs, "f32", oracle, f"row magnitudes M={M}")


def test_gemm_strided_bf16_out(oracle):
    N, K, M = 40, 512, 12
    W, _, s_ref, p_ref = oracle_problem(oracle, tb.INT2, N, K, seed=900)
    Xfull = synth.activations(K + 64, seed=901, M=M)
    X = Xfull[:, :K]
    Y64, Yabs = oracle.gemm64(p_ref, tb.INT2, s_ref, u16(X.contiguous()), N, K)
    Ybuf = torch.zeros((M, N + 24), dtype=torch.bfloat16, device=DEV)
    # keep every device buffer referenced while the raw pointers are in use
    pd, sd, xd = to_dev_packed(p_ref), to_dev_bits(s_ref), Xfull.to(DEV)
    ws = tb.workspace(tb.workspace_bytes(M, N, K), DEV)
    rc = tb.load().tb_gemm(pd.data_ptr(), tb.INT2, sd.data_ptr(), xd.data_ptr(), K + 64, Ybuf.data_ptr(), tb.BF16,
                           N + 24, M, N, K, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert_within(Ybuf[:, :N], Y64, Yabs, "bf16", oracle, "gemm strided")
    assert torch.all(Ybuf[:, N:] == 0)


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("M", [65, 100, 128, 161])
def test_gemm_prefill_blocks(oracle, grid, M):
    """Batches above 64 rows run in one launch as blocks of 128 batch rows
    (M = 65, 100: one ragged block; 161: a full block and a ragged one of
    33 rows; rows past M are never stored)."""
    N, K = 80, 768
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=3100 + M)
    X = synth.activations(K, seed=3200 + M, M=M)
    Y64, Yabs = oracle.gemm64(p_ref, grid, s_ref, u16(X), N, K)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K)
    assert_within(Y, Y64, Yabs, "f32", oracle, f"prefill M={M} grid {grid}")


def test_gemm_prefill_strided_bf16_out(oracle):
    N, K, M = 200, 1024, 130
    W, _, s_ref, p_ref = oracle_problem(oracle, tb.INT3, N, K, seed=3300)
    Xfull = synth.activations(K + 64, seed=3301, M=M)
    X = Xfull[:, :K]
    Y64, Yabs = oracle.gemm64(p_ref, tb.INT3, s_ref, u16(X.contiguous()), N, K)
    Ybuf = torch.zeros((M, N + 24), dtype=torch.bfloat16, device=DEV)
    pd, sd, xd = to_dev_packed(p_ref), to_dev_bits(s_ref), Xfull.to(DEV)
    ws = tb.workspace(tb.workspace_bytes(M, N, K), DEV)
    rc = tb.load().tb_gemm(pd.data_ptr(), tb.INT3, sd.data_ptr(), xd.data_ptr(), K + 64, Ybuf.data_ptr(), tb.BF16,
                           N + 24, M, N, K, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert_within(Ybuf[:, :N], Y64, Yabs, "bf16", oracle, "prefill strided")
    assert torch.all(Ybuf[:, N:] == 0)


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("M", [16, 33, 64])
def test_gemm_multi_tile_split(oracle, grid, M):
    """Several 128-row tiles, a ragged last tile and a 16-way K split."""
    N, K = 300, 2048
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=1100 + M + grid)
    X = synth.activations(K, seed=1200 + M, M=M)
    Y64, Yabs = oracle.gemm64(p_ref, grid, s_ref, u16(X), N, K)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K)
    assert_within(Y, Y64, Yabs, "f32", oracle, f"gemm tiles M={M}")
    assert tb.wait_timeouts() == 0


@pytest.mark.parametrize("grid", [tb.INT2, tb.INT3])
def test_gemm_no_split(oracle, grid):
    """Enough tiles that every CTA covers the whole K range (no K split)."""
    N, K, M = 296 * 128, 256, 20
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=1300 + grid)
    X = synth.activations(K, seed=1301, M=M)
    Y64, Yabs = oracle.gemm64(p_ref, grid, s_ref, u16(X), N, K)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K, out_dtype=torch.bfloat16)
    assert_within(Y, Y64, Yabs, "bf16", oracle, "gemm no split")
    assert tb.wait_timeouts() == 0


@pytest.mark.parametrize("grid", [tb.INT2, tb.INT3])
@pytest.mark.parametrize("M", [4, 16, 64])
def test_gemm_config4_gate_sampled(oracle, grid, M):
    """Qwen3-14B-like gate projection (17408 x 5120) at full size, in the
    launch configuration the benchmark times; 96 sampled rows per batch row
    (tile and split boundaries included) against the oracle."""
    N, K = 17408, 5120
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=4000 + grid)
    X = synth.activations(K, seed=4100 + M, M=M)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K).cpu()
    rng = np.random.default_rng(M + 10 * grid)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 129, N - 128, N - 1], rng.integers(0, N, 90)]))
    Xb = u16(X)
    for m in range(M):
        y64, yabs = oracle.gemv_rows64(p_ref, grid, s_ref, Xb[m], K, rows)
        assert_within(Y[m, rows], y64, yabs, "f32", oracle, f"gate M={M} m={m}")
    assert tb.wait_timeouts() == 0


# ------------------------------------------------------------------ activations

def _x_case(kind, K, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(K, generator=g)
    if kind == "wide_range":       # 2^-60 .. 2^40 inside every group
        e = torch.randint(-60, 41, (K,), generator=g).float()
        x = x.sign() * torch.exp2(e) * (1 + torch.rand(K, generator=g))
    elif kind == "zero_groups":    # whole groups of zeros, one lone value
        x[128:384] = 0
        x[512:640] = 0
        x[600] = 3.0
    elif kind == "subnormal":      # bf16 subnormals and tiny normals mixed with ordinary values
        x[::2] = x[::2] * 2.0 ** -130
    elif kind == "large":
        x = x * 2.0 ** 100
    elif kind == "one_hot":
        x = torch.zeros(K)
        x[777] = -2.5
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("kind", ["wide_range", "zero_groups", "subnormal", "large", "one_hot"])
@pytest.mark.parametrize("api", APIS)
def test_gemv_activation_ranges(oracle, grid, kind, api):
    N, K = 96, 1024
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=1200 + grid)
    x = _x_case(kind, K, 77)
    y64, yabs = oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K)
    y = gemv_via(api, to_dev_packed(p_ref), grid, to_dev_bits(s_ref), x.to(DEV), N, K,
                 torch.empty(N, dtype=torch.float32, device=DEV))
    assert_within(y, y64, yabs, "f32", oracle, f"{kind} {api}")


def test_layer_overlap_flag_and_shared_workspace(oracle):
    """Back-to-back grouped launches sharing one workspace, with and without
    programmatic overlap, give the same bits as each layer launched alone
    with its own workspace, and stay within tolerance of the oracle."""
    shapes = synth.qwen3_layer_shapes(384, 1024, kv_dim=128)
    layers = []
    for L in range(3):
        items = []
        for i, (name, N, K) in enumerate(shapes):
            grid = (tb.INT3, tb.INT2, tb.TERNARY)[(i + L) % 3]
            W = synth.gaussian_weights(N, K, seed=3000 + 10 * L + i).to(DEV)
            s, p, _ = gpu_quantize(W, grid)
            x = synth.activations(K, seed=3100 + 10 * L + i).to(DEV)
            y = torch.empty(N, dtype=torch.float32, device=DEV)
            items.append((p, grid, s, x, y, N, K))
        layers.append(items)
    alone = []
    for it in layers:
        tb.tb_layer_gemv(it)
        torch.cuda.synchronize()
        alone.append([y.clone() for (_, _, _, _, y, _, _) in it])
    # oracle check of the first layer (weights read back from the generator, packed by the oracle)
    for i, (p, grid, s_, x, y, N, K) in enumerate(layers[0]):
        W = synth.gaussian_weights(N, K, seed=3000 + i)
        s_ref = oracle.scales_absmax(W.numpy(), grid)
        p_ref, _ = oracle.pack(W.numpy(), grid, s_ref)
        y64, yabs = oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K)
        assert_within(alone[0][i], y64, yabs, "f32", oracle, f"layer0 item {i}")
    ws = tb.workspace(max(tb.layer_workspace_bytes(tb.linear_items(it)) for it in layers), DEV)
    for flags in (0, tb.FLAG_OVERLAP_PREVIOUS):
        for it in layers:
            for (_, _, _, _, y, _, _) in it:
                y.fill_(float("nan"))
        for it in layers:
            tb.tb_layer_gemv(it, ws=ws, flags=flags)
        torch.cuda.synchronize()
        for L, it in enumerate(layers):
            for i, (p, grid, s, x, y, N, K) in enumerate(it):
                assert torch.equal(y, alone[L][i]), (flags, L, i)


@pytest.mark.parametrize("grid", [tb.INT2, tb.INT3])
def test_gemv_ranges_over_several_tiles(oracle, grid):
    """A tall matrix whose CTA ranges each cover more than one tile (K = 8192:
    64 groups per row, 157 tiles of 256 rows): sampled rows (tile edges,
    ends, random) against the oracle, and the output bit for bit against a
    second launch with programmatic overlap."""
    N, K = 40000, 8192
    W = synth.gaussian_weights(N, K, seed=3500 + grid)
    s_ref = oracle.scales_absmax(w_np(W), grid)
    p_ref, _ = oracle.pack(w_np(W), grid, s_ref)
    x = synth.activations(K, seed=3600 + grid)
    rng = np.random.default_rng(grid)
    rows = np.unique(np.concatenate([[0, 1, N - 1], np.arange(255, N, 256 * 16), rng.integers(0, N, 48)]))
    y64, yabs = oracle.gemv_rows64(p_ref, grid, s_ref, u16(x), K, rows)
    pd, sd, xd = to_dev_packed(p_ref), to_dev_bits(s_ref), x.to(DEV)
    y = torch.empty(N, dtype=torch.float32, device=DEV)
    tb.tb_layer_gemv([(pd, grid, sd, xd, y, N, K)])
    y2 = torch.empty_like(y)
    tb.tb_layer_gemv([(pd, grid, sd, xd, y2, N, K)], flags=tb.FLAG_OVERLAP_PREVIOUS)
    assert tb.sync_status() == 0
    assert torch.equal(y, y2)
    assert_within(y[torch.from_numpy(rows).to(DEV)], y64, yabs, "f32", oracle, f"tall grid {grid}")


@pytest.mark.parametrize("grid", [tb.INT2, tb.INT3])
@pytest.mark.parametrize("tiles_less", [1, 0])
def test_gemv_both_cta_layouts(oracle, grid, tiles_less):
    """A call of 8 chunks per SM or more runs two CTAs per SM, a smaller one
    one CTA: a 2-bit matrix of K = 8192 (16 chunks per 256-row tile) with
    SMs / 2 tiles sits exactly at the switch, one tile fewer just below it
    (3 bits: twice the chunks, both above).  Sampled rows (tile edges, ends,
    random) against the oracle."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    K = 8192
    N = 256 * (sms // 2 - tiles_less) - 17  # ragged last tile
    W = synth.gaussian_weights(N, K, seed=3700 + grid + tiles_less)
    s_ref = oracle.scales_absmax(w_np(W), grid)
    p_ref, _ = oracle.pack(w_np(W), grid, s_ref)
    x = synth.activations(K, seed=3800 + grid)
    rng = np.random.default_rng(7 + grid)
    rows = np.unique(np.concatenate([[0, 1, N - 1], np.arange(255, N, 256 * 8), rng.integers(0, N, 40)]))
    y64, yabs = oracle.gemv_rows64(p_ref, grid, s_ref, u16(x), K, rows)
    y = tb.tb_gemv(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), x.to(DEV), N, K)
    assert tb.sync_status() == 0
    assert_within(y[torch.from_numpy(rows).to(DEV)], y64, yabs, "f32", oracle, f"{N}x{K} grid {grid}")


def test_zz_no_bounded_wait_gave_up():
    """After every test above: no device-side bounded wait (TMA copies,
    tensor-core hand-offs) timed out, so every result above is a real one."""
    torch.cuda.synchronize()
    assert tb.wait_timeouts() == 0


@pytest.mark.parametrize("grid", [tb.INT2, tb.INT3])
@pytest.mark.parametrize("M", [256, 1000])
def test_gemm_prefill_gate_sampled(oracle, grid, M):
    """Prefill at the Qwen3-14B-like gate shape (17408 x 5120), M = 256 and
    1000 batch rows (8 blocks of 128, the last ragged): 64 sampled output
    rows (tile boundaries included) for 24 sampled batch rows (block
    boundaries included) against the oracle."""
    N, K = 17408, 5120
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=4000 + grid)
    X = synth.activations(K, seed=4500 + M, M=M)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K).cpu()
    rng = np.random.default_rng(M + 7 * grid)
    rows = np.unique(np.concatenate([[0, 127, 128, N - 129, N - 128, N - 1], rng.integers(0, N, 58)]))
    ms = np.unique(np.concatenate([[0, 63, 64, 127, 128, M - 1], rng.integers(0, M, 20)]))
    Xb = u16(X)
    for m in ms:
        y64, yabs = oracle.gemv_rows64(p_ref, grid, s_ref, Xb[m], K, rows)
        assert_within(Y[m, rows], y64, yabs, "f32", oracle, f"prefill gate M={M} m={m}")
    assert tb.wait_timeouts() == 0


@pytest.mark.parametrize("grid", [tb.TERNARY, tb.INT3])
def test_gemm_prefill_largest_batch(oracle, grid):
    """The largest batch one tb_gemm call takes, M = 65536 (512 blocks of 128
    batch rows), over a ragged 200-row matrix of two groups: sampled batch
    rows (block boundaries included) against the oracle, all outputs."""
    N, K, M = 200, 256, 65536
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=5100 + grid)
    X = synth.activations(K, seed=5200 + grid, M=M)
    Y = tb.tb_gemm(to_dev_packed(p_ref), grid, to_dev_bits(s_ref), X.to(DEV), N, K).cpu()
    rng = np.random.default_rng(5300 + grid)
    ms = np.unique(np.concatenate([[0, 127, 128, 32767, 32768, M - 129, M - 128, M - 1], rng.integers(0, M, 24)]))
    rows = np.arange(N)
    Xb = u16(X)
    for m in ms:
        y64, yabs = oracle.gemv_rows64(p_ref, grid, s_ref, Xb[m], K, rows)
        assert_within(Y[m], y64, yabs, "f32", oracle, f"M=65536 m={m}")
    assert tb.wait_timeouts() == 0


@pytest.mark.parametrize("grid", [tb.INT2, tb.INT3])
def test_gemm_prefill_is_deterministic(oracle, grid):
    """Units split between CTAs are combined in CTA order: two prefill calls
    on the same inputs give bitwise the same result (and a third, after a
    call of another shape through the same workspace, too)."""
    N, K, M = 4096, 5120, 300
    W, _, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=5400 + grid)
    X = synth.activations(K, seed=5500 + grid, M=M).to(DEV)
    p, s = to_dev_packed(p_ref), to_dev_bits(s_ref)
    ws = tb.workspace(max(tb.workspace_bytes(M, N, K), tb.workspace_bytes(77, N, K)), DEV)
    y1 = tb.tb_gemm(p, grid, s, X, N, K, ws=ws)
    y2 = tb.tb_gemm(p, grid, s, X, N, K, ws=ws)
    tb.tb_gemm(p, grid, s, X[:77].contiguous(), N, K, ws=ws)
    y3 = tb.tb_gemm(p, grid, s, X, N, K, ws=ws)
    assert torch.equal(y1, y2) and torch.equal(y1, y3)
    assert tb.wait_timeouts() == 0
