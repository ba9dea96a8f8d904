"""Host logic of chunked / context-parallel prefill (CPU only, no kernels).

The window ring of a range, the argument checks of the range compressor, and the two
collectives of context-parallel prefill (the halo each rank receives from its predecessor
and the all-gather of compressed entries) over a world-size-2 gloo group on 127.0.0.1.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from compressed_sparse_mqa_dsv4_b200 import cp


def test_window_ring_places_position_j_in_slot_j_mod_R():
    B, n, c, wwin = 2, 6, 3, 4
    for p0 in (0, 2, 17):
        local = torch.arange(B * n * c, dtype=torch.float32).reshape(B, n, c) + 1000
        halo = -torch.arange(B * 5 * c, dtype=torch.float32).reshape(B, 5, c) - 1
        ring, R = cp.window_ring(local, p0, wwin, halo if p0 else None)
        h = min(p0, wwin - 1)
        assert R == h + n and ring.shape == (B, R, c)
        for j in range(p0 - h, p0 + n):
            want = local[:, j - p0] if j >= p0 else halo[:, 5 - (p0 - j)]
            assert torch.equal(ring[:, j % R], want), (p0, j)


def test_window_ring_requires_the_halo():
    with pytest.raises(ValueError):
        cp.window_ring(torch.zeros(1, 4, 2), 8, 4, None)


def test_compress_range_checks_start_and_halo():
    C = torch.zeros(1, 8, 4)
    with pytest.raises(ValueError):
        cp.compress_range(C, C, torch.zeros(2, 4, 2), 4, True, 6)      # start not on a block
    with pytest.raises(ValueError):
        cp.compress_range(C, C, torch.zeros(2, 4, 2), 4, True, 8)      # CSA halo missing


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, n, c = 2, 8, 3
        x = (torch.arange(B * n * c, dtype=torch.float32).reshape(B, n, c) + 100 * rank)
        halo = cp.exchange_halo(x, 4)
        e = torch.full((B, 2, c), float(rank))
        g = cp.allgather_rows(e)
        q.put((rank, halo, g))
    finally:
        dist.destroy_process_group()


def test_halo_and_entry_gather_over_gloo():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, halo, g = q.get(timeout=120)
        out[r] = (halo, g)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    B, n, c = 2, 8, 3
    base = torch.arange(B * n * c, dtype=torch.float32).reshape(B, n, c)
    assert torch.equal(out[0][0], torch.zeros(B, 4, c))                 # rank 0: nothing before it
    assert torch.equal(out[1][0], base[:, n - 4:])                      # rank 1: rank 0's tail
    for r in range(world):
        g = out[r][1]
        assert g.shape == (B, 4, c)
        assert torch.equal(g[:, :2], torch.zeros(B, 2, c)) and torch.equal(g[:, 2:], torch.ones(B, 2, c))
