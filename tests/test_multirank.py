"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The mixer shards by independent sequences, so the benchmark runs one replica
per rank with no collective on the data path; the only cross-rank steps are the
barriers around the timed region and the max-over-ranks reduction of the time.
"""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_setup(world)
    try:
        assert (r, w) == (rank, world)
        bench.barrier(w)
        m = bench.max_over_ranks(float(10 + rank), w)
        q.put((rank, m))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_barrier_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=5) for _ in range(world))
    assert got == [(r, float(10 + world - 1)) for r in range(world)]


def test_byte_accounting_matches_the_layout():
    sys.path.insert(0, ROOT)
    import bench
    # q, k: 2*128 B each; v, o: 2*128 B each; a, b: 4 B each
    assert bench.prefill_bytes_per_token_head(128, 128) == 4 * 256 + 8
    assert bench.prefill_bytes_per_token_head(128, 256) == 2 * 256 + 2 * 512 + 8
    # decode: fp32 state read and written once, plus the token's vectors
    assert bench.decode_bytes_per_head_state(128, 128) == 2 * 65536 + 1024 + 8
    assert bench.prefill_state_bytes(2, 3, 128, 64, True, False) == 2 * 3 * 128 * 64 * 4
