"""The multi-rank path on CPU: two gloo ranks split a batch into row slabs, each
quantizes its slab with the oracle, and the gathered result equals the
single-process quantization; the step time is the max over ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from block_scaled_gemm_rfq_b200.sharding import row_slab


def test_row_slabs_tile_the_batch():
    for M in [1, 127, 128, 255, 256, 257, 1000, 4096, 4097]:
        for world in [1, 2, 3, 4, 8]:
            slabs = [row_slab(M, r, world) for r in range(world)]
            assert slabs[0][0] == 0 and slabs[-1][1] == M
            for (a0, a1), (b0, b1) in zip(slabs, slabs[1:]):
                assert a1 == b0
            for a0, a1 in slabs:
                assert a0 % 256 == 0 or a0 == M
            tiles = [(a1 - a0 + 255) // 256 for a0, a1 in slabs]
            assert max(tiles) - min(tiles) <= 1


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    from block_scaled_gemm_rfq_b200 import workloads as wl
    from block_scaled_gemm_rfq_b200.sharding import max_over_ranks, row_slab
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bits = wl.random_matrix(600, 256, seed=9, scale=3.0)
        a, b = row_slab(600, rank, world)
        mine = oracle.quantize_bf16(bits[a:b], residual=True)
        flat = np.concatenate([mine[k].reshape(-1) for k in ("codes_x", "scales_x", "codes_r", "scales_r")])
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([flat.size], dtype=torch.int64))
        n = max(int(s.item()) for s in sizes)
        buf = torch.zeros(n, dtype=torch.uint8)
        buf[: flat.size] = torch.from_numpy(flat)
        got = [torch.zeros(n, dtype=torch.uint8) for _ in range(world)]
        dist.all_gather(got, buf)
        t = max_over_ranks(10.0 + rank)
        q.put((rank, [g[: int(s.item())].numpy() for g, s in zip(got, sizes)], t))
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(300)
def test_two_gloo_ranks_reassemble_the_batch(oracle):
    import oracle as orc
    from block_scaled_gemm_rfq_b200 import workloads as wl
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    bits = wl.random_matrix(600, 256, seed=9, scale=3.0)
    full = orc.quantize_bf16(bits, residual=True)
    for rank, parts, t in results:
        assert t == 11.0                       # max over ranks of 10 + rank
        pieces = {k: [] for k in ("codes_x", "scales_x", "codes_r", "scales_r")}
        for r, part in enumerate(parts):
            a, b = row_slab(600, r, world)
            rows = b - a
            sizes = [rows * 128, rows * 8, rows * 128, rows * 8]
            offs = np.cumsum([0] + sizes)
            for k, o0, o1 in zip(pieces, offs[:-1], offs[1:]):
                pieces[k].append(part[o0:o1])
        for k in pieces:
            np.testing.assert_array_equal(np.concatenate(pieces[k]), full[k].reshape(-1))
