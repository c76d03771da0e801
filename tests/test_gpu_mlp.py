"""The decode-order decoder layer: q/k/v in one launch on one shared input
(activation records prepared once per code width), then the MLP with gate
and up in one launch whose epilogue writes the down projection's input
h = bf16(silu(gate) * up), then down on h, at Qwen3-8B-like shapes (hidden
4096, MLP 12288) with the grids of layer 0 of the benchmark's stack.

The oracle computes gate and up exactly (fp64), h from them (fp64 silu,
reading R9), and down from its own bf16 rounding of h.  The tolerance of h
follows from the products' bound through silu (|silu'| < 1.1) and the bf16
rounding:
    dg = 1e-5 A_g + 2^-24 |g|        (A = sum |x c s|, the GEMV bound)
    tol_h = 1.01 (1.1 dg (|u| + du) + |silu(g)| du) + 4e-3 |h|
and the down projection's from tol_h through W_down:
    tol_y = A_down(tol_h + 2^-8 |h|) + 1e-5 A_down(|h| + tol_h + 2^-8 |h|) + 2^-24 |y|
where A_down(v) = sum_k |c_k s_k| v_k.  Nothing the oracle or the
tolerance uses comes from the GPU."""
import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth
from decode_gemv_tb_b200 import tb
from tests.helpers import assert_within, u16

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tb.load()


def packed(oracle, m):
    W = synth.gaussian_weights(m.N, m.K, seed=m.seed, dtype=torch.bfloat16)
    s_ref = oracle.scales_absmax(u16(W), m.grid)
    p_ref, _ = oracle.pack(u16(W), m.grid, s_ref)
    p = torch.from_numpy(p_ref.reshape(-1).view(np.uint8).copy()).to(DEV)
    s = torch.from_numpy(s_ref.view(np.int16).copy()).to(DEV).view(torch.bfloat16)
    return p_ref, s_ref, p, s


def bf16_up(v):
    """bf16 bit patterns of values >= v (v >= 0): round to bf16, then one ulp up."""
    b = torch.from_numpy(np.asarray(v, dtype=np.float32)).to(torch.bfloat16)
    bits = b.view(torch.int16).numpy().view(np.uint16).astype(np.uint32) + 1
    return bits.astype(np.uint16)


def test_decode_order_layer(oracle):
    mats = {m.name.split(".")[1]: m for m in synth.config3_stack()[0]}
    x = synth.activations(4096, seed=7001)            # the layer input (after the norm)
    xo = synth.activations(4096, seed=7002)           # stand-in for the attention output
    x2 = synth.activations(4096, seed=7003)           # the MLP input (after the second norm)
    P = {name: packed(oracle, m) for name, m in mats.items()}
    xd, xod, x2d = x.to(DEV), xo.to(DEV), x2.to(DEV)
    ys = {name: torch.full((m.N,), 7.0, dtype=torch.float32, device=DEV) for name, m in mats.items()}

    # q, k, v: one launch, one shared x
    qkv = [(P[n][2], mats[n].grid, P[n][3], xd, ys[n], mats[n].N, mats[n].K) for n in ("q", "k", "v")]
    tb.tb_layer_gemv(qkv)
    tb.tb_layer_gemv([(P["o"][2], mats["o"].grid, P["o"][3], xod, ys["o"], mats["o"].N, mats["o"].K)])
    # gate, up -> h
    N, K = mats["gate"].N, mats["gate"].K
    h = torch.full((N,), 7.0, dtype=torch.bfloat16, device=DEV)
    tb.tb_gate_up_silu((P["gate"][2], mats["gate"].grid, P["gate"][3], x2d, ys["gate"], N, K),
                       (P["up"][2], mats["up"].grid, P["up"][3], x2d, ys["up"], N, K), h)
    # down on the GPU's h
    md = mats["down"]
    tb.tb_layer_gemv([(P["down"][2], md.grid, P["down"][3], h, ys["down"], md.N, md.K)])
    assert tb.sync_status() == 0

    ins = {"q": x, "k": x, "v": x, "o": xo, "gate": x2, "up": x2}
    ref = {}
    for name, xi in ins.items():
        m = mats[name]
        ref[name] = oracle.gemv64(P[name][0], m.grid, P[name][1], u16(xi), m.N, m.K)
        assert_within(ys[name], *ref[name], "f32", oracle, f"decode-order {name}")

    (g, Ag), (u, Au) = ref["gate"], ref["up"]
    h64 = oracle.swiglu64(g, u)
    dg = 1e-5 * Ag + 2.0 ** -24 * np.abs(g)
    du = 1e-5 * Au + 2.0 ** -24 * np.abs(u)
    sg = np.abs(h64 / np.where(u == 0, 1.0, u))  # |silu(g)|
    sg[u == 0] = np.abs(np.array([oracle.silu(a) for a in g[u == 0]]))
    tol_h = 1.01 * (1.1 * dg * (np.abs(u) + du) + sg * du) + 4e-3 * np.abs(h64)
    got_h = h.float().cpu().numpy().astype(np.float64)
    bad = np.nonzero(~(np.abs(got_h - h64) <= tol_h))[0]
    assert bad.size == 0, f"h: {bad.size} out of tolerance, first {bad[:5]}"

    # down: the oracle on its own rounding of h; tolerance propagated from tol_h
    h_ref = oracle.f32_to_bf16_bits(h64.astype(np.float32))
    y_ref, A_ref = oracle.gemv64(P["down"][0], md.grid, P["down"][1], h_ref, md.N, md.K)
    v = tol_h + 2.0 ** -8 * np.abs(h64)
    A_v = oracle.gemv64(P["down"][0], md.grid, P["down"][1], bf16_up(v), md.N, md.K)[1]
    A_h = oracle.gemv64(P["down"][0], md.grid, P["down"][1], bf16_up(np.abs(h64) + v), md.N, md.K)[1]
    tol_y = A_v + 1e-5 * A_h + 2.0 ** -24 * np.abs(y_ref)
    got_y = ys["down"].cpu().numpy().astype(np.float64)
    bad = np.nonzero(~(np.abs(got_y - y_ref) <= tol_y))[0]
    assert bad.size == 0, f"down: {bad.size} out of tolerance, first {bad[:5]}"


def test_gate_up_pair_matches_separate_launches(oracle):
    """The pair's gate and up outputs are those of the grouped launch of the
    same two items, bit for bit (same kernel, same partition)."""
    mats = {m.name.split(".")[1]: m for m in synth.config3_stack()[1]}
    x2d = synth.activations(4096, seed=7101).to(DEV)
    N, K = mats["gate"].N, mats["gate"].K
    pg, pu = packed(oracle, mats["gate"]), packed(oracle, mats["up"])
    yg, yu = torch.empty(N, device=DEV), torch.empty(N, device=DEV)
    h = torch.empty(N, dtype=torch.bfloat16, device=DEV)
    tb.tb_gate_up_silu((pg[2], mats["gate"].grid, pg[3], x2d, yg, N, K), (pu[2], mats["up"].grid, pu[3], x2d, yu, N, K),
                       h)
    yg2, yu2 = torch.empty(N, device=DEV), torch.empty(N, device=DEV)
    tb.tb_layer_gemv([(pg[2], mats["gate"].grid, pg[3], x2d, yg2, N, K), (pu[2], mats["up"].grid, pu[3], x2d, yu2, N, K)])
    assert tb.sync_status() == 0
    assert torch.equal(yg, yg2) and torch.equal(yu, yu2)
    # h is silu(gate) * up of those values, rounded once
    g, u = yg.double(), yu.double()
    want = (g / (1 + torch.exp(-g)) * u)
    assert torch.all((h.double() - want).abs() <= 4e-3 * want.abs() + 1e-30)
