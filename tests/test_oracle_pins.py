"""Pins of the CPU oracle to facts that do not come from the oracle itself:
the ThinkBit page's format facts, hand-worked layout examples, exact
rational arithmetic, library routines (torch bf16 conversion, numpy
matmul), closed forms and invariants.  CPU only."""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from decode_gemv_tb_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
GRIDS = (0, 1, 2)
NAME2GRID = {"ternary": 0, "int2": 1, "int3": 2}
B3 = 3                # the ternary grid in the optional 5-trits-per-byte layout
LAYOUTS = GRIDS + (B3,)


def page_facts():
    facts = {}
    with open(os.path.join(GOLDEN, "page_facts.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val, _ = [p.strip() for p in line.split(";", 2)]
            facts[key] = val
    return facts


def f32_bits(v: float) -> int:
    return int(np.array([v], dtype=np.float32).view(np.uint32)[0])


def bf16_of(v: float) -> int:
    """bf16 bit pattern via torch's conversion (a library routine)."""
    return int(torch.tensor([v], dtype=torch.float32).to(torch.bfloat16).view(torch.int16)[0]) & 0xFFFF


def bf16_value(bits: int) -> float:
    return float(np.array([bits << 16], dtype=np.uint32).view(np.float32)[0])


def rne_fraction(q: Fraction) -> int:
    """Round half to even on an exact rational (Python's round() on a
    Fraction is exact and rounds ties to even)."""
    return round(q)


# ---------------------------------------------------------------- grids

def test_grids_are_the_pages(oracle):
    facts = page_facts()
    for name, grid in NAME2GRID.items():
        want = [int(v) for v in facts[f"grid.{name}"].split(",")]
        assert list(range(oracle.GRID_RANGE[grid][0], oracle.GRID_RANGE[grid][1] + 1)) == want
        one = bf16_of(1.0)
        # every grid point is reached from w = c exactly with s = 1
        got = [oracle.quantize(float(c), one, grid)[0] for c in want]
        assert got == want
        # far outside the grid clamps to its ends
        assert oracle.quantize(1e30, one, grid)[0] == want[-1]
        assert oracle.quantize(-1e30, one, grid)[0] == want[0]


def test_group_size_and_bytes_closed_form(oracle):
    facts = page_facts()
    g = int(facts["group_size"])
    sbits = int(facts["scale_bits"])
    assert oracle.GROUP == g
    for grid, bits in ((0, 2), (1, 2), (2, 3)):
        for N, K in ((1, 128), (3, 256), (256, 1024), (2048, 6144), (17408, 5120)):
            total_bits = 8 * oracle.packed_bytes(grid, N, K) + sbits * N * (K // g)
            # (b + 16/128) bits per weight: 2.125 for the 2-bit container, 3.125 for 3 bits
            assert total_bits == N * K * bits + N * K * sbits // g
            assert total_bits / (N * K) == bits + sbits / g


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_round_matches_torch(oracle):
    rng = np.random.default_rng(1)
    vals = list(rng.standard_normal(4000).astype(np.float32))
    vals += list((rng.standard_normal(2000) * 1e-39).astype(np.float32))  # subnormals
    vals += [0.0, -0.0, 1.0, -1.0, 3.4e38, -3.4e38, float("inf"), float("-inf"), 1e-45, 65504.0]
    # exact ties between two bf16 neighbours, both parities
    for base in (0x3F80, 0x3F81, 0x4000, 0x4001, 0x0001, 0x7F7F):
        vals.append(np.array([(base << 16) | 0x8000], dtype=np.uint32).view(np.float32)[0])
    arr = np.array(vals, dtype=np.float32)
    ours = oracle.f32_to_bf16_bits(arr)
    ref = torch.from_numpy(arr).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert oracle.f32_to_bf16_bits(np.array([np.nan], np.float32))[0] & 0x7F80 == 0x7F80


# ---------------------------------------------------------------- RTN quantize

def _exact_code(w: float, sbits: int, grid: int) -> int:
    lo, hi = (-1, 1) if grid == 0 else ((-2, 1) if grid == 1 else (-4, 3))
    q = Fraction(float(np.float32(w))) / Fraction(bf16_value(sbits))
    return min(hi, max(lo, rne_fraction(q)))


def test_quantize_matches_exact_rational_rounding(oracle):
    rng = np.random.default_rng(2)
    for grid in GRIDS:
        for _ in range(3000):
            s = bf16_of(float(abs(rng.standard_normal()) * 10 ** rng.uniform(-6, 3)) + 1e-30)
            w = float(np.float32(rng.standard_normal() * bf16_value(s) * 3))
            assert oracle.quantize(w, s, grid) == (_exact_code(w, s, grid), 0)


def test_quantize_ties_go_to_even(oracle):
    # w = (k + 1/2) s exactly representable: must round to the even neighbour
    for grid in GRIDS:
        lo, hi = oracle.GRID_RANGE[grid]
        for sv in (1.0, 0.5, 0.015625, 3.0, 0.375, 1.5e-3):
            s = bf16_of(sv)
            sval = bf16_value(s)
            for k2 in range(2 * lo - 1, 2 * hi + 2, 2):  # odd multiples of s/2
                w = k2 * sval / 2
                assert float(np.float32(w)) == w
                want = min(hi, max(lo, round(Fraction(k2, 2))))
                assert want % 2 == 0 or want in (lo, hi)
                assert oracle.quantize(w, s, grid)[0] == want, (grid, sv, k2)
            # one float above / below the tie leaves the even choice
            w = 0.5 * sval
            up = float(np.nextafter(np.float32(w), np.float32(np.inf)))
            dn = float(np.nextafter(np.float32(w), np.float32(0)))
            assert oracle.quantize(up, s, grid)[0] == min(hi, 1)
            assert oracle.quantize(dn, s, grid)[0] == 0


def test_quantize_nonfinite_rules(oracle):
    one = bf16_of(1.0)
    for grid in GRIDS:
        lo, hi = oracle.GRID_RANGE[grid]
        assert oracle.quantize(float("nan"), one, grid) == (0, 1)
        assert oracle.quantize(float("inf"), one, grid) == (hi, 1)
        assert oracle.quantize(float("-inf"), one, grid) == (lo, 1)
        for bad_s in (0x0000, 0x8000, bf16_of(-1.0), 0x7F80, 0x7FC0):
            assert oracle.quantize(0.7, bad_s, grid) == (0, 1)
        # a subnormal scale is valid
        assert oracle.quantize(bf16_value(0x0001) * 1.0, 0x0001, grid) == (min(hi, 1), 0)


# ---------------------------------------------------------------- layout

def _parse_codes(field: str, n: int):
    field = field.strip()
    if "*" in field:
        v, cnt = field.split("*")
        out = [int(v)] * int(cnt)
    else:
        out = [int(v) for v in field.split(",")]
    assert len(out) == n
    return out


def test_format_golden_examples(oracle):
    n_lines = 0
    with open(os.path.join(GOLDEN, "format_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            gname, codes, words, _why = [p.strip() for p in line.split(";", 3)]
            grid = NAME2GRID[gname]
            K = 32 if grid == 2 else 16
            c = _parse_codes(codes, K)
            want = [int(w, 16) for w in words.split(",")]
            # build a one-row, 128-wide problem whose first word/block is the example
            row = np.array(c * (128 // K), dtype=np.float32)[None, :]
            scales = np.full((1, 1), bf16_of(1.0), np.uint16)
            packed, bad = oracle.pack(row, grid, scales)
            assert bad == 0
            got = [int(v) for v in packed[0, : len(want)]]
            assert got == want, (line, [hex(v) for v in got])
            assert list(oracle.unpack(packed, grid, 1, 128)[0, :K]) == c
            n_lines += 1
    assert n_lines >= 20


@pytest.mark.parametrize("grid", GRIDS)
def test_exact_reconstruction_roundtrip(oracle, grid):
    """w = c * s is stored exactly: packing c*s with scale s gives back c."""
    lo, hi = oracle.GRID_RANGE[grid]
    rng = np.random.default_rng(10 + grid)
    N, K = 7, 384
    c = rng.integers(lo, hi + 1, size=(N, K)).astype(np.int64)
    sb = np.array([[bf16_of(float(abs(rng.standard_normal()) * 0.02 + 1e-3)) for _ in range(K // 128)]
                   for _ in range(N)], dtype=np.uint16)
    svals = np.vectorize(bf16_value)(sb).astype(np.float64)
    W = (c * np.repeat(svals, 128, axis=1)).astype(np.float32)
    assert np.array_equal(W.astype(np.float64), c * np.repeat(svals, 128, axis=1))  # exact in fp32
    packed, bad = oracle.pack(W, grid, sb)
    assert bad == 0
    assert packed.shape == (N, (3 * K // 32) if grid == 2 else K // 16)
    assert np.array_equal(oracle.unpack(packed, grid, N, K).astype(np.int64), c)


def test_every_2bit_word_pattern_roundtrips(oracle):
    """All 4^16 patterns cannot be enumerated; cover every (position, code)
    pair plus random words, each through pack and back."""
    rng = np.random.default_rng(3)
    for grid in GRIDS:
        lo, hi = oracle.GRID_RANGE[grid]
        per = 32 if grid == 2 else 16
        rows = []
        for pos in range(per):
            for v in range(lo, hi + 1):
                r = [lo] * 128
                r[pos] = v
                rows.append(r)
        for _ in range(64):
            rows.append(list(rng.integers(lo, hi + 1, size=128)))
        W = np.array(rows, dtype=np.float32)
        packed, _ = oracle.pack(W, grid, np.full((len(rows), 1), bf16_of(1.0), np.uint16))
        assert np.array_equal(oracle.unpack(packed, grid, len(rows), 128), W.astype(np.int8))
        # one-hot rows: the packed row differs from the all-lo row in one word only
        base = packed[0]
        for i, r in enumerate(rows[: per * (hi - lo + 1)]):
            diff = np.nonzero(packed[i] != base)[0]
            pos = i // (hi - lo + 1)
            assert diff.size <= (3 if grid == 2 else 1)
            if diff.size:
                word = pos // 16 if grid != 2 else 3 * (pos // 32) + diff[0] % 3
                assert diff[0] // (3 if grid == 2 else 1) == pos // per


# ---------------------------------------------------------------- 5 trits per byte

def _parse_segments(field: str):
    out = []
    for seg in field.split("|"):
        seg = seg.strip()
        if "*" in seg:
            v, cnt = seg.split("*")
            out += [int(v)] * int(cnt)
        else:
            out += [int(v) for v in seg.split(",")]
    return out


def test_b3_golden_examples(oracle):
    n_lines = 0
    with open(os.path.join(GOLDEN, "format_b3_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            codes, words, _why = [p.strip() for p in line.split(";", 2)]
            c = _parse_segments(codes)
            K = len(c)
            assert K in (128, 256)
            packed, bad = oracle.pack(np.array(c, np.float32)[None, :], B3,
                                      np.full((1, K // 128), bf16_of(1.0), np.uint16))
            assert bad == 0
            assert [int(v) for v in packed[0]] == [int(w, 16) for w in words.split(",")], line
            assert list(oracle.unpack(packed, B3, 1, K)[0]) == c
            n_lines += 1
    assert n_lines >= 12


def test_b3_every_byte_value_decodes_base3(oracle):
    """Each byte value 0..255 written straight into the packed row decodes,
    digit by digit, to Python's floor(v / 3^i) mod 3, minus 1; the other
    bytes (zero) decode to -1 and the row padding is never read."""
    K = 128
    rw = oracle.row_words(B3, K)
    assert rw == 8  # 26 bytes padded to 32
    for b, ndig in ((0, 5), (3, 5), (7, 5), (24, 5), (25, 3)):
        rows = np.zeros((256, rw), np.uint32)
        for v in range(256):
            rows[v, b // 4] = v << (8 * (b % 4))
        rows[:, 7] = 0xFFFFFFFF  # padding bytes 28..31
        codes = oracle.unpack(rows, B3, 256, K)
        for v in range(256):
            assert list(codes[v, 5 * b: 5 * b + ndig]) == [(v // 3 ** i) % 3 - 1 for i in range(ndig)]
            assert np.all(np.delete(codes[v], range(5 * b, 5 * b + ndig)) == -1)


def test_b3_pack_is_a_bijection_on_digit_patterns(oracle):
    """All 3^5 patterns of a full byte pack to the distinct values 0..242,
    each the base-3 number of its digits c + 1; all 3^3 patterns of the
    last byte to 0..26."""
    import itertools
    ones = None
    for first, n, byte in ((10, 5, 2), (125, 3, 25)):
        pats = list(itertools.product((-1, 0, 1), repeat=n))
        rows = np.full((len(pats), 128), -1.0, np.float32)
        for r, pat in enumerate(pats):
            rows[r, first:first + n] = pat
        ones = np.full((len(pats), 1), bf16_of(1.0), np.uint16)
        packed, bad = oracle.pack(rows, B3, ones)
        assert bad == 0
        vals = [(int(packed[r, byte // 4]) >> (8 * (byte % 4))) & 0xFF for r in range(len(pats))]
        assert sorted(vals) == list(range(3 ** n))
        for pat, v in zip(pats, vals):
            assert v == sum((d + 1) * 3 ** i for i, d in enumerate(pat))


def test_b3_bytes_closed_form(oracle):
    facts = page_facts()
    g, sbits = int(facts["group_size"]), int(facts["scale_bits"])
    assert 25 * 5 + 3 == g           # 25 full bytes and one of three trits hold a group
    assert 8 / 5 >= math.log2(3)     # 5 trits fit a byte: 3^5 = 243 <= 256
    assert 3 ** 5 <= 256 < 3 ** 6
    for N, K in ((1, 128), (3, 256), (5, 640), (256, 1024), (2048, 6144), (17408, 5120)):
        G = K // g
        assert oracle.packed_bytes(B3, N, K) == N * 16 * math.ceil(26 * G / 16)
        bits = (8 * oracle.packed_bytes(B3, N, K) + sbits * N * G) / (N * K)
        assert bits <= 2 + sbits / g      # never above the 2-bit container
        if G % 8 == 0:                   # 8 groups = 208 bytes = 13 x 16: no padding
            assert bits == 26 * 8 / g + sbits / g == 1.75


def test_b3_quantizes_and_scales_like_ternary(oracle):
    rng = np.random.default_rng(90)
    for _ in range(2000):
        s = bf16_of(float(abs(rng.standard_normal()) * 10 ** rng.uniform(-6, 3)) + 1e-30)
        w = float(np.float32(rng.standard_normal() * bf16_value(s) * 3))
        assert oracle.quantize(w, s, B3) == (_exact_code(w, s, 0), 0)
    one = bf16_of(1.0)
    assert oracle.quantize(float("nan"), one, B3) == (0, 1)
    assert oracle.quantize(float("inf"), one, B3) == (1, 1)
    assert oracle.quantize(float("-inf"), one, B3) == (-1, 1)
    for bad_s in (0x0000, 0x8000, bf16_of(-1.0), 0x7F80, 0x7FC0):
        assert oracle.quantize(0.7, bad_s, B3) == (0, 1)
    W = (rng.standard_normal((6, 384)) * 0.02).astype(np.float32)
    t = torch.from_numpy(W).view(6, 3, 128).abs().amax(-1)  # ternary divisor |qmin| = 1
    assert np.array_equal(oracle.scales_absmax(W, B3), t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))


@pytest.mark.parametrize("K", [128, 384, 640, 1024])
def test_b3_exact_reconstruction_roundtrip(oracle, K):
    rng = np.random.default_rng(100 + K)
    N = 7
    c = rng.integers(-1, 2, size=(N, K)).astype(np.int64)
    sb = np.array([[bf16_of(float(abs(rng.standard_normal()) * 0.02 + 1e-3)) for _ in range(K // 128)]
                   for _ in range(N)], dtype=np.uint16)
    svals = np.vectorize(bf16_value)(sb).astype(np.float64)
    W = (c * np.repeat(svals, 128, axis=1)).astype(np.float32)
    packed, bad = oracle.pack(W, B3, sb)
    assert bad == 0
    assert packed.shape == (N, 4 * math.ceil(26 * (K // 128) / 16))
    assert np.array_equal(oracle.unpack(packed, B3, N, K).astype(np.int64), c)
    # the padding words past 26 G bytes stay zero
    tail = packed.view(np.uint8).reshape(N, -1)[:, 26 * (K // 128):]
    assert not tail.any()


# ---------------------------------------------------------------- scales

@pytest.mark.parametrize("grid", GRIDS)
def test_scales_absmax_against_torch(oracle, grid):
    rng = np.random.default_rng(20 + grid)
    N, K = 9, 512
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[3, 128:256] = 0.0  # an all-zero group
    got = oracle.scales_absmax(W, grid)
    d = {0: 1.0, 1: 2.0, 2: 4.0}[grid]  # |qmin| of the page's grid
    t = torch.from_numpy(W).view(N, K // 128, 128).abs().amax(-1) / d
    ref = t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    ref[ref == 0] = bf16_of(1.0)
    assert np.array_equal(got, ref)
    # bf16 weights take the same path after exact widening
    Wb = torch.from_numpy(W).to(torch.bfloat16)
    got_b = oracle.scales_absmax(Wb.view(torch.int16).numpy().view(np.uint16), grid)
    tb = Wb.float().view(N, K // 128, 128).abs().amax(-1) / d
    ref_b = tb.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()
    ref_b[ref_b == 0] = bf16_of(1.0)
    assert np.array_equal(got_b, ref_b)


def test_scale_rule_edges_golden(oracle):
    """The non-finite and overflow branches of the scale rule against
    hand-worked values (tests/golden/scale_examples.txt): NaN and +-Inf
    entries are skipped, a zero scale becomes 1.0, one that rounds to
    infinity becomes the largest finite bf16."""
    names = {"ternary": 0, "int2": 1, "int3": 2}
    n = 0
    for line in open(os.path.join(GOLDEN, "scale_examples.txt")):
        if not line.strip() or line.startswith("#"):
            continue
        grid_s, entries, want, _ = [f.strip() for f in line.split(";", 3)]
        group = np.zeros(128, dtype=np.float32)
        i = 0
        for e in entries.split(","):
            v, cnt = e.strip().split(" x")
            group[i:i + int(cnt)] = np.float32(float(v))
            i += int(cnt)
        got = oracle.scales_absmax(group.reshape(1, 128), names[grid_s])
        assert int(got[0, 0]) == int(want, 16), line
        n += 1
    assert n == 13


def test_scales_reach_grid_ends(oracle):
    """With absmax/|qmin| scales, the group's most negative entry lands on
    qmin exactly (it is -|qmin| * s before rounding)."""
    rng = np.random.default_rng(5)
    for grid in GRIDS:
        lo, hi = oracle.GRID_RANGE[grid]
        W = (rng.standard_normal((4, 256)) * 0.02).astype(np.float32)
        W[:, 7] = -np.abs(W).max(axis=1) * 2  # a clear negative maximum in group 0
        s = oracle.scales_absmax(W, grid)
        packed, _ = oracle.pack(W, grid, s)
        codes = oracle.unpack(packed, grid, 4, 256)
        # bf16 rounding of the scale may move the quotient by < 1/2 code
        assert np.all(codes[:, 7] == lo)
        assert codes.min() >= lo and codes.max() <= hi


# ---------------------------------------------------------------- products

def _random_problem(oracle, grid, N, K, seed):
    rng = np.random.default_rng(seed)
    lo, hi = oracle.GRID_RANGE[grid]
    c = rng.integers(lo, hi + 1, size=(N, K))
    sb = np.array([[bf16_of(float(abs(rng.standard_normal()) * 0.02 + 1e-3)) for _ in range(K // 128)]
                   for _ in range(N)], dtype=np.uint16)
    svals = np.vectorize(bf16_value)(sb).astype(np.float64)
    W64 = c * np.repeat(svals, 128, axis=1)
    packed, _ = oracle.pack(W64.astype(np.float32), grid, sb)
    xb = np.array([bf16_of(float(v)) for v in rng.standard_normal(K)], dtype=np.uint16)
    return c, sb, W64, packed, xb


@pytest.mark.parametrize("grid", LAYOUTS)
def test_gemv_equals_dense_matmul(oracle, grid):
    """Textbook reduction: y equals numpy's matmul of the dequantized
    matrix (built here directly as c*s, not by the oracle) with x."""
    N, K = 37, 640
    c, sb, W64, packed, xb = _random_problem(oracle, grid, N, K, 30 + grid)
    x64 = oracle.bf16_bits_to_f32(xb).astype(np.float64)
    y, yabs = oracle.gemv64(packed, grid, sb, xb, N, K)
    ref = W64 @ x64
    assert np.all(np.abs(y - ref) <= 1e-12 * np.abs(W64) @ np.abs(x64))
    assert np.allclose(yabs, np.abs(W64) @ np.abs(x64), rtol=1e-12, atol=0)


def test_gemv_integer_exact(oracle):
    """Integer x and power-of-two scales: y is an exact integer multiple of
    the scale, equal to an int64 matmul."""
    rng = np.random.default_rng(40)
    for grid in LAYOUTS:
        lo, hi = oracle.GRID_RANGE[grid]
        N, K = 19, 1024
        c = rng.integers(lo, hi + 1, size=(N, K)).astype(np.int64)
        xi = rng.integers(-8, 9, size=K).astype(np.int64)
        e = int(rng.integers(-12, 3))
        sb = np.full((N, K // 128), bf16_of(2.0 ** e), np.uint16)
        packed, _ = oracle.pack((c * 2.0 ** e).astype(np.float32), grid, sb)
        xb = np.array([bf16_of(float(v)) for v in xi], dtype=np.uint16)
        y, _ = oracle.gemv64(packed, grid, sb, xb, N, K)
        assert np.array_equal(y, (c @ xi).astype(np.float64) * 2.0 ** e)


def test_gemv_permutation_rows(oracle):
    """Codes forming a permutation pattern with unit scales pick single
    entries of x: y[n] = x[p(n)].  Non-square, so a transposed operand or
    a wrong row stride fails."""
    rng = np.random.default_rng(50)
    for grid in LAYOUTS:
        N, K = 24, 384
        p = rng.permutation(K)[:N]
        c = np.zeros((N, K))
        c[np.arange(N), p] = 1
        sb = np.full((N, K // 128), bf16_of(1.0), np.uint16)
        packed, _ = oracle.pack(c.astype(np.float32), grid, sb)
        xb = np.array([bf16_of(float(v)) for v in rng.standard_normal(K)], dtype=np.uint16)
        y, _ = oracle.gemv64(packed, grid, sb, xb, N, K)
        assert np.array_equal(y, oracle.bf16_bits_to_f32(xb)[p].astype(np.float64))


def test_gemv_group_locality(oracle):
    """x zero outside group j: y depends on scale column j only, linearly."""
    grid = 2
    N, K = 11, 512
    c, sb, W64, packed, xb = _random_problem(oracle, grid, N, K, 60)
    j = 2
    xl = xb.copy()
    xl[: 128 * j] = 0
    xl[128 * (j + 1):] = 0
    y0, _ = oracle.gemv64(packed, grid, sb, xl, N, K)
    s2 = sb.copy()
    s2[:, [0, 1, 3]] = bf16_of(7.0)  # other groups' scales do not matter
    y1, _ = oracle.gemv64(packed, grid, s2, xl, N, K)
    assert np.array_equal(y0, y1)
    s3 = sb.copy()
    s3[:, j] = np.array([bf16_of(2 * bf16_value(int(v))) for v in sb[:, j]], np.uint16)
    y2, _ = oracle.gemv64(packed, grid, s3, xl, N, K)
    assert np.array_equal(y2, 2 * y0)


def test_gemv_linearity(oracle):
    N, K = 13, 256
    c, sb, W64, packed, xb = _random_problem(oracle, 1, N, K, 70)
    y, _ = oracle.gemv64(packed, 1, sb, xb, N, K)
    x2 = np.array([bf16_of(2 * v) for v in oracle.bf16_bits_to_f32(xb)], np.uint16)
    y2, _ = oracle.gemv64(packed, 1, sb, x2, N, K)
    assert np.array_equal(y2, 2 * y)


def test_gemm_rows_are_gemvs(oracle):
    N, K, M = 21, 384, 5
    c, sb, W64, packed, xb = _random_problem(oracle, 2, N, K, 80)
    rng = np.random.default_rng(81)
    Xb = np.array([[bf16_of(float(v)) for v in rng.standard_normal(K)] for _ in range(M)], np.uint16)
    Y, Yabs = oracle.gemm64(packed, 2, sb, Xb, N, K)
    for m in range(M):
        y, yabs = oracle.gemv64(packed, 2, sb, Xb[m], N, K)
        assert np.array_equal(Y[m], y) and np.array_equal(Yabs[m], yabs)
    X64 = oracle.bf16_bits_to_f32(Xb).astype(np.float64)
    assert np.all(np.abs(Y - X64 @ W64.T) <= 1e-12 * np.abs(X64) @ np.abs(W64.T))
    rows = np.array([20, 0, 7])
    yr, _ = oracle.gemv_rows64(packed, 2, sb, Xb[1], K, rows)
    assert np.array_equal(yr, Y[1, rows])


def test_output_rounding(oracle):
    y = np.array([1.0 + 2 ** -30, -3.0000001, 1e-40, 0.0])
    assert np.array_equal(oracle.round_out(y, "f32"), y.astype(np.float32))
    ref = torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16).float().numpy()
    assert np.array_equal(oracle.round_out(y, "bf16"), ref)


# ---------------------------------------------------------------- workloads

def test_workload_mix_matches_page():
    facts = page_facts()
    want = {0: float(facts["mix.ternary_pct"]), 1: float(facts["mix.int2_pct"]), 2: float(facts["mix.int3_pct"])}
    for stack in (synth.config3_stack(), synth.config5_stack()):
        fr = synth.grid_fractions(stack)
        for g in GRIDS:
            assert abs(100 * fr[g] - want[g]) < 0.25, (g, fr)
        for mats in stack:
            for m in mats:
                if m.name.endswith((".q", ".k")):
                    assert m.grid in (1, 2)  # 2 bits or more
    # Config 5 packed size: 3.82 GB scale (2.125 / 3.125 bits per weight with scales)
    tot = sum(m.N * m.K * (3.125 if m.grid == 2 else 2.125) / 8 for mats in synth.config5_stack() for m in mats)
    assert 3.75e9 < tot < 3.9e9


# ---------------------------------------------------------------- gated MLP input (reading R9)

def test_silu_against_high_precision(oracle):
    """silu(g) = g / (1 + e^-g) in fp64 against a 60-digit decimal
    evaluation (correctly rounded exp at that precision, independent of the
    C library): within 4 ulps, and the special values exactly."""
    import decimal
    ctx = decimal.Context(prec=60)
    pts = [-100.0, -30.0, -20.0, -5.0, -1.0, -0.25, -2.0 ** -20, 0.0, 2.0 ** -20, 0.5, 1.0, 2.0, 7.25, 30.0, 100.0]
    for g in pts:
        D = decimal.Decimal(g)
        ref = float(ctx.divide(D, ctx.add(decimal.Decimal(1), ctx.exp(-D))))
        got = oracle.silu(g)
        assert abs(got - ref) <= 4 * np.spacing(abs(ref)) + 1e-300, (g, got, ref)
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu(800.0) == 800.0          # e^-800 underflows: g / 1
    assert oracle.silu(-800.0) == 0.0           # e^800 overflows: g / inf -> -0
    # the function's shape: silu(g) - silu(-g) = g (since e^-g / (1 + e^-g) + 1 / (1 + e^-g) = 1)
    for g in (0.3, 1.7, 4.0):
        assert abs((oracle.silu(g) - oracle.silu(-g)) - g) <= 4 * np.spacing(g)


def test_swiglu_is_silu_times_up(oracle):
    rng = np.random.default_rng(31)
    g = rng.standard_normal(257) * 3
    u = rng.standard_normal(257)
    h = oracle.swiglu64(g, u)
    assert np.array_equal(h, np.array([oracle.silu(a) * b for a, b in zip(g, u)]))
    assert np.array_equal(oracle.swiglu64(g, 2 * u), 2 * h)   # exact scaling
    assert np.all(oracle.swiglu64(g, np.zeros_like(u)) == 0)
