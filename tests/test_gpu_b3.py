"""The optional 5-trits-per-byte ternary layout on the GPU against the CPU
oracle, through the C interface: scales, pack and unpack bit-exact; GEMV,
GEMM rows and grouped layer items within |y - y_ref| <= 1e-5 sum|x w|
(fp32) or that plus 4e-3 |y_ref| (bf16).  The oracle packs from the same
weights itself; nothing it consumes comes from the GPU."""
import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth
from decode_gemv_tb_b200 import tb
from tests.helpers import assert_within, u16, u32, w_np
from tests.test_gpu_parity import DEV, gpu_quantize, oracle_problem, to_dev_bits, to_dev_packed

pytestmark = pytest.mark.gpu
B3 = tb.TERNARY_B3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tb.load()


@pytest.mark.parametrize("wdt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(1, 128), (5, 256), (37, 640), (256, 1024), (300, 2048), (64, 3200)])
def test_b3_scales_pack_unpack_bitexact(oracle, wdt, shape):
    N, K = shape
    W = synth.gaussian_weights(N, K, seed=N * 11 + K, dtype=wdt).to(DEV)
    s, p, bad = gpu_quantize(W, B3)
    assert p.numel() == tb.packed_bytes(B3, N, K) == oracle.packed_bytes(B3, N, K)
    ws = w_np(W)
    s_ref = oracle.scales_absmax(ws, B3)
    assert np.array_equal(u16(s), s_ref)
    p_ref, bad_ref = oracle.pack(ws, B3, s_ref)
    assert np.array_equal(u32(p).reshape(p_ref.shape), p_ref)
    assert bad == bad_ref == 0
    assert np.array_equal(tb.tb_unpack(p, B3, N, K).cpu().numpy(), oracle.unpack(p_ref, B3, N, K))


def test_b3_pack_edge_values(oracle):
    """Ties, clamps, NaN/Inf weights, invalid and tiny scales, in every
    byte position of a group (the short last byte included)."""
    rng = np.random.default_rng(17)
    N, K = 8, 256
    sv = np.array([1.0, 0.5, 3.0, 0.375, 1e-20, 2.0 ** -126, 0.0, -1.0, np.inf, np.nan, 1e-38, 7.0e-39,
                   0.015625, 1.5e-3, 2.0 ** -135, 4.0], dtype=np.float32).reshape(N, 2)
    s = torch.from_numpy(sv).to(torch.bfloat16)
    sval = s.float().numpy()
    W = np.empty((N, K), dtype=np.float32)
    for n in range(N):
        for j in range(2):
            base = sval[n, j] if np.isfinite(sval[n, j]) and sval[n, j] > 0 else 1.0
            k2 = rng.integers(-5, 6, size=128)  # multiples of s/2 around the ternary grid: ties and clamps
            blk = (k2 * np.float64(base) / 2).astype(np.float32)
            blk[::7] = np.nextafter(blk[::7], np.float32(np.inf))
            blk[::11] = np.nextafter(blk[::11], np.float32(-np.inf))
            blk[5], blk[6], blk[9], blk[126], blk[127] = np.nan, np.inf, -np.inf, np.nan, -np.inf
            W[n, 128 * j:128 * (j + 1)] = blk
    bad = torch.zeros(1, dtype=torch.int32, device=DEV)
    p = tb.tb_pack(torch.from_numpy(W).to(DEV), B3, s.to(DEV), bad_count=bad)
    p_ref, bad_ref = oracle.pack(W, B3, u16(s))
    assert np.array_equal(u32(p).reshape(p_ref.shape), p_ref)
    assert int(bad.item()) == bad_ref > 0
    Wb = torch.from_numpy(W).to(torch.bfloat16)
    pb = tb.tb_pack(Wb.to(DEV), B3, s.to(DEV))
    pb_ref, _ = oracle.pack(u16(Wb), B3, u16(s))
    assert np.array_equal(u32(pb).reshape(pb_ref.shape), pb_ref)


def test_b3_unpack_any_bytes(oracle):
    """Random bytes, the never-written values 243..255 included, decode
    digit by digit exactly as the oracle's rule says."""
    N, K = 33, 1152
    g = torch.Generator().manual_seed(23)
    raw = torch.randint(0, 256, (tb.packed_bytes(B3, N, K),), generator=g, dtype=torch.int32).to(torch.uint8)
    raw[:256] = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    codes = tb.tb_unpack(raw.to(DEV), B3, N, K)
    ref = oracle.unpack(raw.numpy().view(np.uint32).reshape(N, -1), B3, N, K)
    assert np.array_equal(codes.cpu().numpy(), ref)


@pytest.mark.parametrize("shape", [(1, 128), (7, 256), (15, 384), (16, 1152), (17, 640), (33, 1024), (100, 2048),
                                   (9, 3200), (65, 4096), (70, 6144), (3, 57600)])
@pytest.mark.parametrize("out", ["f32", "bf16"])
def test_b3_gemv_parity(oracle, shape, out):
    """Group counts below, at and above 32 (several rows per warp, ragged
    lanes, several groups per lane) and the largest supported K."""
    N, K = shape
    W, x, s_ref, p_ref = oracle_problem(oracle, B3, N, K, seed=N * 13 + K)
    y64, yabs = oracle.gemv64(p_ref, B3, s_ref, u16(x), N, K)
    s, p, _ = gpu_quantize(W.to(DEV), B3)
    guard = 64
    ybuf = torch.full((N + guard,), 123.25, dtype=torch.float32 if out == "f32" else torch.bfloat16, device=DEV)
    y = ybuf[:N]
    tb.tb_gemv(p, B3, s, x.to(DEV), N, K, y=y)
    assert_within(y, y64, yabs, out, oracle, f"b3 gemv {shape}")
    assert torch.all(ybuf[N:] == 123.25), "wrote past the end of y"


@pytest.mark.parametrize("case", [c for c in synth.config2_cases() if c.grid == tb.TERNARY], ids=lambda m: m.name)
def test_b3_gemv_config2_shapes(oracle, case):
    """The Qwen3-1.7B-like shapes of the ternary cases, in the 5-trit layout."""
    N, K = case.N, case.K
    W, x, s_ref, p_ref = oracle_problem(oracle, B3, N, K, seed=case.seed)
    y64, yabs = oracle.gemv64(p_ref, B3, s_ref, u16(x), N, K)
    y = tb.tb_gemv(to_dev_packed(p_ref), B3, to_dev_bits(s_ref), x.to(DEV), N, K)
    assert_within(y, y64, yabs, "f32", oracle, case.name + "_b3")


def test_b3_gemv_integer_exact_bitwise(oracle):
    N, K = 48, 1024
    g = torch.Generator().manual_seed(199)
    c = torch.randint(-1, 2, (N, K), generator=g)
    x = torch.randint(-8, 9, (K,), generator=g).to(torch.bfloat16)
    s = torch.full((N, K // 128), 2.0 ** -5, dtype=torch.bfloat16)
    p_ref, _ = oracle.pack((c.float() * 2.0 ** -5).numpy(), B3, u16(s))
    y64, _ = oracle.gemv64(p_ref, B3, u16(s), u16(x), N, K)
    y = tb.tb_gemv(to_dev_packed(p_ref), B3, s.to(DEV), x.to(DEV), N, K)
    assert np.array_equal(y.cpu().numpy(), y64.astype(np.float32))


def test_b3_gemm_rows_strided_bf16(oracle):
    N, K, M = 40, 512, 5
    W, _, s_ref, p_ref = oracle_problem(oracle, B3, N, K, seed=2100)
    X = synth.activations(K, seed=2101, M=M)
    Y64, Yabs = oracle.gemm64(p_ref, B3, s_ref, u16(X), N, K)
    Xbuf = torch.zeros((M, K + 8), dtype=torch.bfloat16, device=DEV)
    Xbuf[:, :K] = X.to(DEV)
    Ybuf = torch.zeros((M, N + 24), dtype=torch.bfloat16, device=DEV)
    ws = tb.workspace(tb.workspace_bytes(M, N, K), DEV)
    p, s = to_dev_packed(p_ref), to_dev_bits(s_ref)  # kept alive until the kernels have run
    rc = tb.load().tb_gemm(p.data_ptr(), B3, s.data_ptr(), Xbuf.data_ptr(), K + 8, Ybuf.data_ptr(), tb.BF16, N + 24,
                           M, N, K, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert_within(Ybuf[:, :N], Y64, Yabs, "bf16", oracle, "b3 gemm")
    assert torch.all(Ybuf[:, N:] == 0)


def test_b3_gemm_prefill(oracle):
    N, K, M = 48, 640, 70
    W, _, s_ref, p_ref = oracle_problem(oracle, B3, N, K, seed=2150)
    X = synth.activations(K, seed=2151, M=M)
    Y64, Yabs = oracle.gemm64(p_ref, B3, s_ref, u16(X), N, K)
    Y = tb.tb_gemm(to_dev_packed(p_ref), B3, to_dev_bits(s_ref), X.to(DEV), N, K)
    assert_within(Y, Y64, Yabs, "f32", oracle, "b3 prefill")


def test_b3_layer_items_and_noalloc(oracle):
    """5-trit items mixed into a grouped launch with the other grids; the
    no-workspace entry point on the same matrix."""
    specs = [(tb.INT3, 256, 512), (B3, 192, 512), (tb.INT2, 64, 512), (tb.TERNARY, 320, 1536), (B3, 512, 1536)]
    items, refs = [], []
    for i, (grid, N, K) in enumerate(specs):
        W, x, s_ref, p_ref = oracle_problem(oracle, grid, N, K, seed=2200 + i)
        refs.append(oracle.gemv64(p_ref, grid, s_ref, u16(x), N, K))
        y = torch.empty(N, dtype=torch.float32, device=DEV)
        items.append((to_dev_packed(p_ref), grid, to_dev_bits(s_ref), x.to(DEV), y, N, K))
    tb.tb_layer_gemv(items)
    first = [it[4].clone() for it in items]
    tb.tb_layer_gemv(items)
    for i, it in enumerate(items):
        assert_within(it[4], *refs[i], "f32", oracle, f"layer item {i}")
        assert torch.equal(it[4], first[i])
    p, grid, s, x, _, N, K = items[4]
    y = torch.empty(N, dtype=torch.float32, device=DEV)
    tb.tb_gemv_noalloc(p, grid, s, x, N, K, y)
    assert torch.equal(y, first[4])
