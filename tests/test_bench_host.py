"""bench.py's host-side arithmetic (no GPU): the algorithmic bytes of a
product in every layout, the rule that drops the committed DRAM-traffic
figure once the kernel's sources change, and the `config` object both arms
print."""
import json
import os
import shutil

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    import bench as b
    return b


def test_algo_bytes_every_layout(bench, oracle):
    from decode_gemv_tb_b200 import tb
    for N, K in ((256, 1024), (2048, 6144), (17408, 5120), (3, 640)):
        for grid in (tb.TERNARY, tb.INT2, tb.INT3, tb.TERNARY_B3):
            # packed codes as the oracle lays them out, bf16 scales, bf16 x, fp32 y
            want = oracle.packed_bytes(grid, N, K) + 2 * N * (K // 128) + 2 * K + 4 * N
            assert bench.algo_bytes(N, K, grid) == want, (grid, N, K)
        # batch M: M rows of x and of y
        assert bench.algo_bytes(N, K, tb.INT2, M=8) == oracle.packed_bytes(1, N, K) + 2 * N * (K // 128) \
            + 8 * 2 * K + 8 * 4 * N


def test_traffic_figure_tracks_the_kernel_sources(bench, tmp_path, monkeypatch):
    """A traffic record's ratio is used while the hashed sources are
    unchanged, and dropped (None) as soon as one of them differs or the
    record is missing."""
    import hashlib
    fake = tmp_path / "root"
    (fake / "profiles").mkdir(parents=True)
    srcs = ["decode_gemv_tb_b200/csrc/tb_gemv8.cu", "decode_gemv_tb_b200/csrc/tb_partition.h"]
    h = hashlib.sha256()
    for s in srcs:
        dst = fake / s
        dst.parent.mkdir(parents=True, exist_ok=True)
        shutil.copy(os.path.join(ROOT, s), dst)
        h.update(open(dst, "rb").read())
    monkeypatch.setattr(bench, "ROOT", str(fake))
    assert bench.traffic_per_launch(1000.0) is None  # no record
    rec = {"kernel": "k_gemv8", "traffic_over_algorithmic": 1.0125, "kernel_sources": srcs,
           "kernel_sources_sha256": h.hexdigest()}
    json.dump(rec, open(fake / bench.TRAFFIC_RECORD, "w"))
    assert bench.traffic_per_launch(1000.0) == pytest.approx(1012.5)
    with open(fake / srcs[0], "a") as f:
        f.write("\n")
    assert bench.traffic_per_launch(1000.0) is None
    # the committed record, if any, names existing sources
    committed = os.path.join(ROOT, bench.TRAFFIC_RECORD)
    if os.path.exists(committed):
        for s in json.load(open(committed))["kernel_sources"]:
            assert os.path.exists(os.path.join(ROOT, s))


def test_workload_config_names_the_stack(bench):
    from decode_gemv_tb_b200 import synth
    stack = synth.config3_stack()
    cfg = bench.workload_config(stack, 1)
    assert cfg["batch"] == 1 and cfg["layers"] == 36 and cfg["hidden"] == 4096 and cfg["mlp"] == 12288
    assert cfg["parallelism"] == "replicas1"
    mix = cfg["grid_mix"]
    assert abs(sum(mix.values()) - 1.0) < 1e-3
    # 2.01 GB of algorithmic bytes per step: codes, scales and y of all 252
    # products, and the four input vectors of each layer (q/k/v share one,
    # gate/up another, all of 4096 elements: k, v and up read no bytes of
    # their own)
    every = sum(bench.algo_bytes(m.N, m.K, m.grid) for mats in stack for m in mats)
    step = cfg["step_algorithmic_bytes"]
    assert every - step == 36 * 3 * 2 * 4096
    assert step == sum(bench.layer_algo_bytes(mats) for mats in stack)
    assert 2.0e9 < step < 2.02e9
    roles = [bench.input_role(m) for m in stack[0]]
    assert roles == ["q", "k", "v", "o", "gate", "up", "down"]
