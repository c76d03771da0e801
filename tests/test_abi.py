"""The C interface on the host (no GPU needed): the shared library loads,
exports every entry point include/tb.h declares, computes sizes in closed
form and rejects bad arguments before launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

from decode_gemv_tb_b200 import build as tbbuild
from decode_gemv_tb_b200 import tb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tb.h")


@pytest.fixture(scope="module")
def lib():
    tbbuild.build()
    return tb.load()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*TB_API\s+(?:(?:const|unsigned|signed)\s+)*[a-z_0-9]+\s*\*?\s*(tb_[a-z_0-9]+)\s*\(", src,
                       flags=re.M)
    return sorted(set(names))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("tb_pack", "tb_unpack", "tb_gemv", "tb_gemm", "tb_layer_gemv", "tb_scales_absmax",
                 "tb_packed_bytes", "tb_scale_bytes", "tb_status_string", "tb_version", "tb_workspace_bytes",
                 "tb_layer_workspace_bytes"):
        assert must in names
    assert set(names) == set(tb.SIGNATURES), "binding and header disagree"


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", tb.LIB_PATH], capture_output=True, text=True, check=True)
    exported = {line.split()[-1] for line in out.stdout.splitlines() if " T " in line}
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # nothing but the C interface is exported
    assert {n for n in exported if not n.startswith("tb_")} <= {"_init", "_fini"}


def test_sizes_closed_form(lib):
    for grid, bits in ((0, 2), (1, 2), (2, 3)):
        for N, K in ((1, 128), (256, 1024), (17408, 5120), (5120, 17408)):
            assert tb.packed_bytes(grid, N, K) == N * K * bits // 8
            assert tb.scale_bytes(N, K) == N * (K // 128) * 2
            # 2.125 / 3.125 bits per weight including scales
            assert 8 * (tb.packed_bytes(grid, N, K) + tb.scale_bytes(N, K)) == N * K * (bits + 0.125)
    assert tb.packed_bytes(1, 4, 100) == 0 and tb.packed_bytes(7, 4, 128) == 0 and tb.scale_bytes(0, 128) == 0
    assert lib.tb_version() >= 100
    for s in range(7):
        assert lib.tb_status_string(s)


FAKE = 1 << 40  # a 256-byte-aligned address that is never dereferenced


def test_workspace_sizes(lib):
    al = lambda b: (b + 255) // 256 * 256
    for M, N, K in ((2, 100, 5120), (4, 100, 5120), (16, 17408, 17408), (17, 7, 1024), (31, 64, 128)):
        # below the tensor-core threshold (32) the kernel reads X as it is: no workspace, a nominal 256
        assert tb.workspace_bytes(M, N, K) == 256
    for M, N, K in ((32, 100, 5120), (33, 17408, 5120), (64, 7, 1024), (64, 40000, 4096)):
        # tensor-core path, data only: per group NP rows of X (256 bytes each) in the MMA's layout,
        # NP = M rounded up to 16; the scales transposed per 128-row tile; a counter per tile; K-split
        # partials of NP x 128 fp32 per tile and split; twice that (control words front, data back)
        NP, tiles, G = (M + 15) // 16 * 16, (N + 127) // 128, K // 128
        splits = max(1, min((296 + tiles // 2) // tiles, 16, G))
        data = (al(G * NP * 256) + al(tiles * G * 128 * 2) + al(4 * tiles) +
                (al(tiles * splits * NP * 128 * 4) if splits > 1 else 0))
        assert tb.workspace_bytes(M, N, K) == 2 * data, (M, N, K)
    for M, N, K in ((65, 100, 5120), (256, 17408, 5120), (257, 7, 1024), (65536, 128, 128)):
        # prefill path: per CTA (at most 256, at most one per chunk) a 4-byte flag (control) and 128 rows x
        # 128 fp32 partial sums (data); chunks = tiles of 128 rows x blocks of 128 batch rows x groups
        ctas = min(256, (N + 127) // 128 * -(-M // 128) * (K // 128))
        control, data = al(4 * ctas), al(ctas * 128 * 128 * 4)
        assert tb.workspace_bytes(M, N, K) == 2 * max(control, data), (M, N, K)
    for N, K in ((1, 128), (256, 1024), (17408, 5120), (100, 1408), (4096, 12288)):
        # batch 1: control = 256 flagged 8-byte partial words per CTA (at most 512 CTAs, at most one per
        # chunk of two groups); data = the activation records of x (1088 bytes per group); size
        # 2 max(control, data)
        G, tiles = K // 128, (N + 255) // 256
        ctas = min(512, tiles * -(-G // 2))
        control, data = al(2048 * ctas), al(1088 * G)
        assert tb.workspace_bytes(1, N, K) == 2 * max(control, data)
    assert tb.workspace_bytes(0, 8, 128) == 0 and tb.workspace_bytes(1, 8, 100) == 0
    assert tb.workspace_bytes(65537, 8, 128) == 0 and tb.workspace_bytes(1, 0, 128) == 0
    # a layer: the items together; records once per distinct (x, K, code width)
    X1, X2 = FAKE, FAKE + 4096
    shapes = ((4096, 4096, 2, X1), (1024, 4096, 1, X1), (1024, 4096, 0, X1), (4096, 12288, 0, X1),
              (4096, 4096, 2, X2))  # (N, K, grid, x): k and v share their records, nothing else does
    items = (tb.Linear * len(shapes))()
    for i, (N, K, grid, x) in enumerate(shapes):
        items[i] = tb.Linear(FAKE, FAKE, x, FAKE, N, K, grid, 0)
    tiles = sum((N + 255) // 256 for N, _, _, _ in shapes)
    # chunks of two 3-bit groups or four 2-bit groups per 256-row tile
    chunks = sum((N + 255) // 256 * -(-(K // 128) // (2 if grid == 2 else 4)) for N, K, grid, _ in shapes)
    rec = sum(al(1088 * (K // 128)) for i, (_, K, _, _) in enumerate(shapes) if i != 2)
    control, data = al(2048 * min(512, chunks)), rec
    assert tb.layer_workspace_bytes(items) == 2 * max(control, data)
    # a layer whose records outweigh its control words
    wide = (tb.Linear * 2)()
    wide[0] = tb.Linear(FAKE, FAKE, X1, FAKE, 256, 1 << 17, 1, 0)
    wide[1] = tb.Linear(FAKE, FAKE, X2, FAKE, 256, 1 << 17, 2, 0)
    control, data = al(2048 * 512), 2 * al(1088 * 1024)
    assert data > control and tb.layer_workspace_bytes(wide) == 2 * data


def test_argument_errors_before_launch(lib):
    A = FAKE
    W = 1 << 20  # workspace size, never touched
    # null pointers / bad enums -> TB_ERR_ARG (1)
    assert lib.tb_gemv(0, 1, A, A, A, 0, 16, 128, A, W, 0) == 1
    assert lib.tb_gemv(A, 9, A, A, A, 0, 16, 128, A, W, 0) == 1
    assert lib.tb_gemv(A, 1, A, A, A, 5, 16, 128, A, W, 0) == 1
    assert lib.tb_gemv(A, 1, A, A, A, 0, 16, 128, 0, W, 0) == 1
    assert lib.tb_gemv(A, 1, A, A, A, 0, 16, 128, A, 16, 0) == 1  # workspace too small
    assert lib.tb_pack(A, 3, 16, 128, 1, A, A, 0, 0) == 1
    assert lib.tb_layer_gemv(0, 1, 0, A, W, 0) == 1
    items = (tb.Linear * 17)()
    assert lib.tb_layer_gemv(ctypes.cast(items, ctypes.c_void_p), 17, 0, A, W, 0) == 1
    assert lib.tb_layer_gemv(ctypes.cast(items, ctypes.c_void_p), 0, 0, A, W, 0) == 1
    # shapes -> TB_ERR_SHAPE (2)
    assert lib.tb_gemv(A, 1, A, A, A, 0, 0, 128, A, W, 0) == 2
    assert lib.tb_gemv(A, 1, A, A, A, 0, 16, 100, A, W, 0) == 2
    assert lib.tb_gemv(A, 1, A, A, A, 0, 16, 0, A, W, 0) == 2
    assert lib.tb_gemm(A, 1, A, A, 128, A, 0, 16, 65537, 16, 128, A, 1 << 30, 0) == 2
    assert lib.tb_gemm(A, 1, A, A, 128, A, 0, 16, 0, 16, 128, A, W, 0) == 2
    assert lib.tb_gemm(A, 1, A, A, 120, A, 0, 16, 4, 16, 128, A, W, 0) == 2
    assert lib.tb_gemm(A, 1, A, A, 128, A, 0, 8, 4, 16, 128, A, W, 0) == 2
    assert lib.tb_pack(A, 0, 16, 200, 1, A, A, 0, 0) == 2
    assert lib.tb_unpack(A, 1, -1, 128, A, 0) == 2
    # alignment -> TB_ERR_ALIGN (3)
    assert lib.tb_gemv(A + 8, 1, A, A, A, 0, 16, 128, A, W, 0) == 3
    assert lib.tb_gemv(A, 1, A + 1, A, A, 0, 16, 128, A, W, 0) == 3
    assert lib.tb_gemv(A, 1, A + 8, A, A, 0, 16, 128, A, W, 0) == 3  # scales: 16 bytes
    assert lib.tb_gemv(A, 1, A, A + 2, A, 0, 16, 128, A, W, 0) == 3
    assert lib.tb_gemv(A, 1, A, A, A + 2, 0, 16, 128, A, W, 0) == 3
    assert lib.tb_gemv(A, 1, A, A, A, 0, 16, 128, A + 16, W, 0) == 3
    assert lib.tb_gemm(A, 1, A, A, 132, A, 0, 16, 4, 16, 128, A, W, 0) == 3
    assert lib.tb_pack(A + 4, 0, 16, 128, 1, A, A, 0, 0) == 3
    items = (tb.Linear * 2)()
    for i in range(2):
        items[i] = tb.Linear(A, A, A, A, 16, 128, 1, 0)
    assert lib.tb_layer_gemv(ctypes.cast(items, ctypes.c_void_p), 2, 2, A, W, 0) == 1  # unknown flag
    assert lib.tb_layer_gemv(ctypes.cast(items, ctypes.c_void_p), 2, 0, A + 64, W, 0) == 3
    items[1].x = A + 8
    assert lib.tb_layer_gemv(ctypes.cast(items, ctypes.c_void_p), 2, 0, A, W, 0) == 3
    items[1].x = A
    items[1].K = 130
    assert lib.tb_layer_gemv(ctypes.cast(items, ctypes.c_void_p), 2, 0, A, W, 0) == 2


def test_prefill_workspace_is_bounded(lib):
    """Batches above 64 rows run in one launch, in blocks of 128 batch rows:
    the workspace grows with the chunks only up to the 256-CTA bound, so a
    prefill batch needs no more than 2 x 256 x 128 x 128 x 4 bytes."""
    bound = 2 * 256 * 128 * 128 * 4
    for N, K in ((100, 5120), (17408, 5120), (7, 1024)):
        for M in (65, 97, 100, 130, 4096 + 17, 65536):
            assert 0 < tb.workspace_bytes(M, N, K) <= bound
    assert tb.workspace_bytes(65536, 17408, 5120) == bound
    assert tb.workspace_bytes(65536, 64, 128) > 0 and tb.workspace_bytes(65537, 64, 128) == 0


def test_b3_sizes_and_limits(lib, oracle):
    """The 5-trits-per-byte layout: closed-form row bytes (the oracle's too),
    the shared-memory bound on K, and no workspace for its layer items."""
    import math
    B3 = tb.TERNARY_B3
    for N, K in ((1, 128), (3, 256), (5, 640), (256, 1024), (2048, 6144), (17408, 5120)):
        want = N * 16 * math.ceil(26 * (K // 128) / 16)
        assert tb.packed_bytes(B3, N, K) == want == oracle.packed_bytes(B3, N, K)
    assert tb.packed_bytes(B3, 4, 100) == 0
    A, W = FAKE, 1 << 30  # workspace size, never touched
    big = 128 * 451  # 451 groups of activations do not fit in shared memory
    assert lib.tb_gemv(A, B3, A, A, A, 0, 16, big, A, W, 0) == 4
    assert lib.tb_gemm(A, B3, A, A, big, A, 0, 16, 3, 16, big, A, W, 0) == 4
    assert lib.tb_gemv_noalloc(A, B3, A, A, A, 0, 16, big, 0) == 4
    items = (tb.Linear * 2)()
    items[0] = tb.Linear(A, A, A, A, 16, big, B3, 0)
    items[1] = tb.Linear(A, A, A, A, 64, 1024, 1, 0)
    assert lib.tb_layer_gemv(ctypes.cast(items, ctypes.c_void_p), 2, 0, A, W, 0) == 4
    # a layer's 5-trit items add nothing to its workspace
    one = (tb.Linear * 1)()
    one[0] = items[1]
    items[0].K = 1024
    assert tb.layer_workspace_bytes(items) == tb.layer_workspace_bytes(one) > 0


def test_binding_fails_loudly_without_library(tmp_path):
    saved = tb._lib
    tb._lib = None
    try:
        with pytest.raises(tb.TBError):
            tb.load(str(tmp_path / "missing.so"))
    finally:
        tb._lib = saved


def test_gate_up_workspace_and_errors(lib):
    """tb_gate_up_silu: the batch-1 rule for its two items with the pair's
    flagged gate values (8 N bytes of control words); shape and argument
    errors before any launch."""
    al = lambda b: (b + 255) // 256 * 256
    A, W = FAKE, 1 << 30
    for (N, K, gg, gu) in ((12288, 4096, 2, 0), (17408, 5120, 1, 1), (300, 640, 0, 2)):
        two = (tb.Linear * 2)()
        two[0] = tb.Linear(A, A, A, A, N, K, gg, 0)
        two[1] = tb.Linear(A, A, A, A, N, K, gu, 0)
        g = ctypes.cast(ctypes.byref(two, 0), ctypes.c_void_p)
        u = ctypes.cast(ctypes.byref(two, ctypes.sizeof(tb.Linear)), ctypes.c_void_p)
        G, T = K // 128, (N + 255) // 256
        chunks = sum(T * -(-G // (2 if gr == 2 else 4)) for gr in (gg, gu))
        shared = (gg == 2) == (gu == 2)  # same x: one record set when the code widths agree
        control = al(2048 * min(512, chunks)) + al(8 * N)
        data = al(1088 * G) * (1 if shared else 2)
        assert lib.tb_gate_up_workspace_bytes(g, u) == 2 * max(control, data)
    two = (tb.Linear * 2)()
    two[0] = tb.Linear(A, A, A, A, 64, 1024, 1, 0)
    two[1] = tb.Linear(A, A, A, A, 32, 1024, 1, 0)
    g = ctypes.cast(ctypes.byref(two, 0), ctypes.c_void_p)
    u = ctypes.cast(ctypes.byref(two, ctypes.sizeof(tb.Linear)), ctypes.c_void_p)
    assert lib.tb_gate_up_workspace_bytes(g, u) == 0                 # N differs
    assert lib.tb_gate_up_silu(g, u, A, 0, A, W, 0) == 2               # TB_ERR_SHAPE
    two[1].N = 64
    assert lib.tb_gate_up_silu(g, u, 0, 0, A, W, 0) == 1               # h missing
    assert lib.tb_gate_up_silu(g, u, A, 2, A, W, 0) == 1               # unknown flag
    assert lib.tb_gate_up_silu(g, u, A + 1, 0, A, W, 0) == 3           # h misaligned
    two[1].grid = 3
    assert lib.tb_gate_up_silu(g, u, A, 0, A, W, 0) == 4               # 5-trit layout: not in the pair
