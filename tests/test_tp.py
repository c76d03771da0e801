"""Tensor-parallel sharding (decode_gemv_tb_b200/tp.py) on two gloo ranks on
the CPU.  The format claims are checked directly -- a rank's column shard
is the oracle's pack of its rows of W, a row shard the oracle's pack of its
128-groups -- and the assembled products against the oracle's full product:
row-parallel partials summed by one all_reduce, column-parallel rows
gathered.  The per-rank product here is the oracle itself (the GPU product
is exercised by tests/test_gpu_tp.py)."""
import os
import socket
import sys

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.join(os.path.dirname(__file__), "..")


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_product(oracle):
    def product(packed, grid, scales, x, N, K):
        y64, _ = oracle.gemv64(packed.numpy().view(np.uint32), grid, scales.numpy().view(np.uint16),
                               x.numpy().view(np.uint16), N, K)
        return torch.from_numpy(y64.astype(np.float32))
    return product


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from decode_gemv_tb_b200 import synth, tp
        from oracle import tb_oracle as oracle
        oracle.build()
        product = _oracle_product(oracle)
        ok = 1.0
        for i, (grid, N, K, kind) in enumerate(((2, 300, 1024, "row"), (1, 301, 1152, "row"), (0, 300, 640, "column"),
                                               (2, 257, 512, "column"))):
            W = synth.gaussian_weights(N, K, seed=60 + i).numpy()
            s = oracle.scales_absmax(W, grid)
            p, _ = oracle.pack(W, grid, s)
            x = synth.activations(K, seed=70 + i)
            y64, yabs = oracle.gemv64(p, grid, s, x.view(torch.int16).numpy().view(np.uint16), N, K)
            pt = torch.from_numpy(p.reshape(-1).view(np.uint8).copy())
            st = torch.from_numpy(s.view(np.int16).copy())
            lin = tp.ShardedLinear(pt, st, grid, N, K, kind, dist)
            # the shard is the pack of the sliced weights
            if kind == "row":
                Wl = np.ascontiguousarray(W[:, lin.g0 * 128:lin.g1 * 128])
                p_l, _ = oracle.pack(Wl, grid, oracle.scales_absmax(Wl, grid))
            else:
                Wl = np.ascontiguousarray(W[lin.n0:lin.n1])
                p_l, _ = oracle.pack(Wl, grid, oracle.scales_absmax(Wl, grid))
            ok *= float(np.array_equal(lin.packed.numpy().view(np.uint32), p_l.reshape(-1)))
            y = lin.forward(x.view(torch.int16), product).numpy().astype(np.float64)
            err = np.abs(y - y64)
            ok *= float(np.all(err <= 1e-5 * yabs + 4 * 2.0 ** -24 * yabs))
        out[rank] = ok
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_and_assemble():
    world = 2
    out = torch.zeros(world, dtype=torch.float64).share_memory_()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    assert out.tolist() == [1.0, 1.0]


def test_ranges_cover_exactly():
    sys.path.insert(0, ROOT)
    from decode_gemv_tb_b200 import tp
    for N in (1, 7, 4096, 12289):
        for R in (1, 2, 3, 8):
            rs = [tp.column_range(N, r, R) for r in range(R)]
            assert rs[0][0] == 0 and rs[-1][1] == N and all(a[1] == b[0] for a, b in zip(rs, rs[1:]))
    for K in (128, 640, 12288):
        for R in (1, 2, 4, 8):
            gs = [tp.group_range(K, r, R) for r in range(R)]
            assert gs[0][0] == 0 and gs[-1][1] == K // 128 and all(a[1] == b[0] for a, b in zip(gs, gs[1:]))
