"""Multi-rank host path on CPU: world size 2 over gloo.

The hot path shards without exchange, so the only multi-rank logic is the
replica seeding and the max / sum bookkeeping around the timed region;
both are exercised here with real processes and a real process group.
"""

import os
import socket
import sys

import pytest
import torch.multiprocessing as tmp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    from quantized_paged_kv_tile_b200 import synth
    from quantized_paged_kv_tile_b200.dist import Ranks
    import bench
    r = Ranks(backend="gloo", timeout_s=60)
    try:
        r.barrier()
        w = synth.workload("qwen3_4b", replica=r.rank)
        elapsed = 10.0 + rank            # pretend per-rank timings
        mx = r.max(elapsed)
        bm = bench.byte_model(w, 0, 0)
        total = r.sum(bm["quantize"] + bm["decode"])
        rows = synth.kv_rows(synth.workload("tiny", replica=r.rank), "k", 4)
        q.put((rank, mx, total, w.seed, w.table_seed, rows.float().sum().item()))
        r.barrier()
    finally:
        r.close()


def test_two_rank_max_sum_and_replica_seeds():
    ctx = tmp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(rk, 2, port, q)) for rk in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort()
    (r0, mx0, tot0, s0, t0, x0), (r1, mx1, tot1, s1, t1, x1) = res
    assert mx0 == mx1 == 11.0                       # max over ranks, seen by every rank
    assert tot0 == tot1 and tot0 > 0                # whole-job bytes = sum over ranks
    assert s0 != s1 and t0 != t1 and x0 != x1       # independent replica batches
    import bench
    sys.path.insert(0, ROOT)
    from quantized_paged_kv_tile_b200 import synth
    bm = bench.byte_model(synth.workload("qwen3_4b"), 0, 0)
    assert tot0 == pytest.approx(2 * (bm["quantize"] + bm["decode"]))


def test_byte_model_matches_hand_count():
    # Qwen3-4B-shaped step: 786432 tokens x 8 heads; K and V at 4 bits, T=64:
    # quantize reads 256 B (K+V fp16) and writes 144 B per token-head;
    # decode reads 144 B per token-head of the 12288 full tiles, 4 B per page
    # of table, the one-token tail (6 x 8 x 512 B) and q + out
    sys.path.insert(0, ROOT)
    import bench
    from quantized_paged_kv_tile_b200 import synth
    bm = bench.byte_model(synth.workload("qwen3_4b"), 0, 0)
    tok_heads = 6 * 131072 * 8
    assert bm["quantize"] == tok_heads * (512 + 144)
    assert bm["decode"] == tok_heads * 144 + 6 * 8192 * 4 + 6 * 8 * 512 + 6 * 32 * 128 * 4
    assert bm["append"] == 6 * 8 * 128 * 2 * 2 * 2
