"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on
the same seeded inputs.  Sizes span several tiles, several heads and
sequences, scattered pages and ragged tails; tolerances are the ones stated
in tests/parity_helpers.py."""

import math

import numpy as np
import pytest
import torch

from oracle import kvq_oracle as o
from quantized_paged_kv_tile_b200 import kvq, synth
from quantized_paged_kv_tile_b200.paged import PagedKVCache

from parity_helpers import (ATTN_REL_L2_MAX, TileStats, compare_sequence_tiles, decode_over_gpu_pages, make_cache,
                            oracle_decode_sequence, rel_l2, unpack_all)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kvq.load_library()


def _prefilled(w, device="cuda", num_splits=0, extra_tokens=0):
    cfg, cache = make_cache(w, extra_tokens=extra_tokens, num_splits=num_splits)
    total = int(sum(w.lens))
    rk = synth.kv_rows(w, "k", total, device=device)
    rv = synth.kv_rows(w, "v", total, device=device)
    cache.prefill(rk, rv, w.lens)
    torch.cuda.synchronize()
    assert cache.status() == 0
    return cfg, cache, rk, rv


def _starts(lens):
    return np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)


# ----------------------------------------------------------------- quantize

QUANT_CASES = [
    # (T, bits_k, bits_v, iters, heads, lens)
    (64, 4, 4, 4, 1, (1024,)),              # the tiny workload's shape
    (64, 4, 2, 4, 2, (300, 129, 64)),       # ragged tails, several seqs
    (32, 2, 3, 1, 2, (200, 96)),
    (128, 4, 2, 2, 3, (384, 130)),
    (128, 3, 4, 8, 1, (256,)),
    (64, 2, 2, 0, 2, (192,)),               # n = 0: plain RTN of the rotated tile
    (64, 8, 8, 4, 2, (300, 70)),            # 8-bit codes
    (128, 8, 8, 2, 1, (260,)),
    (32, 8, 8, 1, 1, (100,)),
]


@pytest.mark.parametrize("t,bk,bv,n,h,lens", QUANT_CASES)
def test_quantize_matches_oracle(t, bk, bv, n, h, lens):
    w = synth.workload("prefill_sweep", num_seqs=len(lens), lens=lens, num_kv_heads=h, tile_tokens=t,
                       bits_k=bk, bits_v=bv, iters=n)
    cfg, cache, rk, rv = _prefilled(w)
    rk_h, rv_h = rk.cpu().numpy(), rv.cpu().numpy()
    tiles = [(s, i) for s in range(len(lens)) for i in range(lens[s] // t)]
    sk, sv = TileStats(), TileStats()
    compare_sequence_tiles(cfg, cache, rk_h, rv_h, _starts(lens), tiles, sk, sv)
    sk.check()
    sv.check()
    # tails hold the unfinished tile's raw rows, bit-exact
    kt, vt = cache.k_tail.cpu().numpy(), cache.v_tail.cpu().numpy()
    for s, L in enumerate(lens):
        tau = L % t
        r0 = _starts(lens)[s] + L - tau
        for h_ in range(h):
            np.testing.assert_array_equal(kt[s, h_, :tau], rk_h[r0:r0 + tau, h_])
            np.testing.assert_array_equal(vt[s, h_, :tau], rv_h[r0:r0 + tau, h_])


def test_pages_byte_identical_to_oracle_packing():
    # wherever the GPU and the oracle agree on every code and metadata value
    # of a tile, the page bytes must be the oracle packer's bytes
    w = synth.workload("prefill_sweep", num_seqs=2, lens=(256, 192), num_kv_heads=2, tile_tokens=64, bits_k=4,
                       bits_v=2, iters=4)
    cfg, cache, rk, rv = _prefilled(w)
    rk_h, rv_h = rk.cpu().numpy(), rv.cpu().numpy()
    kp, vp = cache.k_pool.cpu().numpy(), cache.v_pool.cpu().numpy()
    bt = cache.block_tables.cpu().numpy()
    starts = _starts(w.lens)
    tiles = [(s, ti) for s, L in enumerate(w.lens) for ti in range(L // 64)]
    gk, gv = unpack_all(cfg, cache, tiles, False), unpack_all(cfg, cache, tiles, True)
    checked = 0
    for n, (s, ti) in enumerate(tiles):
        blocks = bt[s, ti * 4:(ti + 1) * 4]
        for h in range(2):
            for rows, pool, g, bits, is_v in ((rk_h, kp, gk, 4, False), (rv_h, vp, gv, 2, True)):
                r0 = starts[s] + ti * 64
                ref = o.quantize_tile(rows[r0:r0 + 64, h], bits, 4, dtype=np.float32)
                meta = g["meta"][n, h]
                same = (np.array_equal(g["codes"][n, h], ref["codes"]) and np.array_equal(meta[:, 0], ref["s_t"])
                        and np.array_equal(meta[:, 1], ref["z_t"]) and np.array_equal(g["cvec"][n, h], ref["c_t"]))
                if not same:
                    continue
                want = np.zeros_like(pool)
                o.write_tile_pages(want, blocks, h, ref, bits, 64, is_v)
                for blk in blocks:
                    np.testing.assert_array_equal(pool[blk, h], want[blk, h])
                checked += 1
    assert checked >= 16


def test_degenerate_tiles():
    # all-zero tile, a tile of identical tokens, a tile whose rotated image has
    # 126 exactly-zero channels (the clamp path).  On the last one every row is
    # identical up to rounding after one iteration, so later channel stds are
    # rounding noise next to the clamp eps: which side of eps they land on
    # depends on the summation order, and the split of the scale between R and
    # C is not unique.  Codes and the dequantized tile (the product) are.
    cfg = kvq.Config(num_kv_heads=1, group_size=1, tile_tokens=64, bits_k=4, bits_v=4, iters=8)
    h = o.sylvester_hadamard(128)
    v01 = (h[:, 0] + h[:, 1]) * math.sqrt(128) / 2
    rng = np.random.default_rng(7)
    row = rng.standard_normal(128).astype(np.float16)
    tiles = [np.zeros((64, 128), np.float16), np.tile(row, (64, 1)),
             (np.arange(1, 65)[:, None] * v01[None, :]).astype(np.float16)]
    rows = np.concatenate(tiles)[:, None, :]
    bt = np.arange(12, dtype=np.int32).reshape(1, 12)
    cache = PagedKVCache(cfg, 1, 192, block_table=bt, num_splits=1)
    x = torch.from_numpy(rows).cuda()
    cache.prefill(x, x, [192])
    torch.cuda.synchronize()
    assert cache.status() == 0
    g = unpack_all(cfg, cache, [(0, 0), (0, 1), (0, 2)], False)
    st = TileStats()
    for i, tile in enumerate(tiles):
        ref = o.quantize_tile(tile, 4, 8, dtype=np.float32)
        assert np.all(np.isfinite(g["meta"][i, 0].astype(np.float32)))
        st.add(g["codes"][i, 0], g["meta"][i, 0], g["cvec"][i, 0], g["rot"][i, 0], ref)
        ref_rot, _ = o.dequantize_tile(ref["codes"], ref["s_t"], ref["z_t"], ref["c_t"])
        scale = max(np.abs(ref_rot).max(), 1e-30)
        assert np.abs(g["rot"][i, 0] - ref_rot).max() <= 4e-3 * scale
    assert st.max_code_diff <= 1
    assert not g["rot"][0].any()


def test_bad_block_id_sets_status_and_skips():
    cfg = kvq.Config(num_kv_heads=1, group_size=4, tile_tokens=64, bits_k=4, bits_v=4, iters=1)
    bt = np.arange(8, dtype=np.int32).reshape(1, 8)
    cache = PagedKVCache(cfg, 1, 128, block_table=bt, num_splits=1)
    cache.block_tables[0, 5] = 1000  # outside [0, num_blocks)
    x = torch.randn((128, 1, 128), device="cuda").half()
    before = cache.k_pool.clone()
    cache.prefill(x, x, [128])
    torch.cuda.synchronize()
    assert cache.status() == kvq.KVQ_ERR_DEVICE_BOUNDS
    # the tile with the bad page was skipped, the other one written
    assert torch.equal(cache.k_pool[4:8], before[4:8])
    assert cache.k_pool[0:4].any()


# ------------------------------------------------------------------- decode

DECODE_CASES = [
    # (workload overrides)
    dict(),                                                   # tiny: 1 seq x 1024, g=8, T=64, b=4/4
    dict(lens=(1000,)),                                       # ragged tail (1000 = 15 tiles + 40)
    dict(num_seqs=3, lens=(700, 64, 30), num_kv_heads=2, group_size=4, bits_v=2),
    dict(num_seqs=2, lens=(520, 1), num_kv_heads=2, group_size=1, tile_tokens=128, bits_k=2, bits_v=4, iters=2),
    dict(num_seqs=2, lens=(333, 257), num_kv_heads=1, group_size=3, tile_tokens=32, bits_k=4, bits_v=2, iters=1),
    dict(num_seqs=2, lens=(700, 90), num_kv_heads=2, group_size=4, bits_k=3, bits_v=3),   # 3-bit pages
    dict(num_seqs=1, lens=(600,), num_kv_heads=1, group_size=8, tile_tokens=128, bits_k=3, bits_v=4, iters=2),
]


@pytest.mark.parametrize("over", DECODE_CASES)
def test_decode_matches_oracle(over):
    w = synth.workload("tiny", **over)
    cfg, cache, rk, rv = _prefilled(w)
    q = synth.queries(w, device="cuda")
    out = cache.decode(q)
    torch.cuda.synchronize()
    assert cache.status() == 0
    rk_h, rv_h, q_h = rk.cpu().numpy(), rv.cpu().numpy(), q.cpu().numpy()
    out_h = out.float().cpu().numpy()
    starts = _starts(w.lens)
    for s, L in enumerate(w.lens):
        ref = oracle_decode_sequence(cfg, rk_h[starts[s]:starts[s] + L], rv_h[starts[s]:starts[s] + L], q_h[s])
        for hq in range(w.num_q_heads):
            err = rel_l2(out_h[s, hq], ref[hq])
            assert err <= ATTN_REL_L2_MAX, (s, hq, err)


DECODE_SWEEP = ([(t, bk, bv, g) for t in (32, 64, 128) for bk in (2, 3, 4) for bv in (2, 3, 4) for g in (2, 8)]
                + [(t, 8, 8, g) for t in (32, 64, 128) for g in (2, 8)])


@pytest.mark.parametrize("t,bk,bv,g", DECODE_SWEEP)
def test_decode_sweep_every_instantiation(t, bk, bv, g):
    # every decode template (T, b_K, b_V) with a small and the largest group;
    # 3 full tiles plus a ragged tail, split over 2 chunks.  The decode is
    # held to 1e-3 against attention over the GPU's own pages (read by the
    # oracle), the pages to the quantize bars against the oracle: with 2-bit
    # codes and ~400 tokens one allowed code difference can move the
    # end-to-end output by more than 1e-3 by itself.
    L = 3 * t + 7
    w = synth.workload("tiny", num_seqs=1, lens=(L,), num_kv_heads=1, group_size=g, tile_tokens=t, bits_k=bk,
                       bits_v=bv, iters=1)
    cfg, cache, rk, rv = _prefilled(w, num_splits=2)
    q = synth.queries(w, device="cuda")
    out = cache.decode(q)
    torch.cuda.synchronize()
    assert cache.status() == 0
    ref = decode_over_gpu_pages(cfg, cache, 0, L, q.cpu().numpy()[0])
    out_h = out.float().cpu().numpy()[0]
    for hq in range(g):
        assert rel_l2(out_h[hq], ref[hq]) <= ATTN_REL_L2_MAX, hq
    sk, sv = TileStats(), TileStats()
    compare_sequence_tiles(cfg, cache, rk.cpu().numpy(), rv.cpu().numpy(), [0], [(0, i) for i in range(3)], sk, sv)
    sk.check()
    sv.check()


def test_decode_only_on_oracle_packed_pages():
    # isolate the read path: seeded random codes / metadata packed by the oracle
    rng = np.random.default_rng(99)
    for t, bk, bv, g in ((64, 4, 4, 8), (128, 4, 2, 4), (32, 2, 2, 2)):
        cfg = kvq.Config(num_kv_heads=2, group_size=g, tile_tokens=t, bits_k=bk, bits_v=bv, iters=0)
        lens = [5 * t + 17, 2 * t]
        bps = max(-(-L // 16) for L in lens)
        bt = rng.permutation(2 * bps).astype(np.int32).reshape(2, bps)
        cache = PagedKVCache(cfg, 2, bps * 16, block_table=bt, num_splits=3)
        kp = np.zeros(tuple(cache.k_pool.shape), np.uint8)
        vp = np.zeros(tuple(cache.v_pool.shape), np.uint8)
        k_hat = [[None] * 2 for _ in range(2)]
        v_hat = [[None] * 2 for _ in range(2)]
        kt = np.zeros(tuple(cache.k_tail.shape), np.float16)
        vt = np.zeros(tuple(cache.v_tail.shape), np.float16)
        for s, L in enumerate(lens):
            for h in range(2):
                parts_k, parts_v = [], []
                for ti in range(L // t):
                    blocks = bt[s, ti * t // 16:(ti + 1) * t // 16]
                    for bits, pool, parts, is_v in ((bk, kp, parts_k, False), (bv, vp, parts_v, True)):
                        tile = {"codes": rng.integers(0, 1 << bits, size=(t, 128)).astype(np.uint8),
                                "s_t": rng.uniform(0.02, 0.4, t).astype(np.float16),
                                "z_t": (-rng.uniform(0.2, 3.0, t)).astype(np.float16),
                                "c_t": rng.uniform(0.3, 2.0, 128).astype(np.float16)}
                        o.write_tile_pages(pool, blocks, h, tile, bits, t, is_v)
                        parts.append(o.dequantize_tile(tile["codes"], tile["s_t"], tile["z_t"], tile["c_t"])[1])
                tau = L % t
                kt[s, h, :tau] = rng.standard_normal((tau, 128)).astype(np.float16)
                vt[s, h, :tau] = rng.standard_normal((tau, 128)).astype(np.float16)
                k_hat[s][h] = np.concatenate(parts_k + [kt[s, h, :tau].astype(np.float64)])
                v_hat[s][h] = np.concatenate(parts_v + [vt[s, h, :tau].astype(np.float64)])
        cache.k_pool.copy_(torch.from_numpy(kp))
        cache.v_pool.copy_(torch.from_numpy(vp))
        cache.k_tail.copy_(torch.from_numpy(kt))
        cache.v_tail.copy_(torch.from_numpy(vt))
        cache.seq_lens.copy_(torch.tensor(lens, dtype=torch.int32))
        q = torch.from_numpy(rng.standard_normal((2, 2 * g, 128)).astype(np.float16)).cuda()
        out = cache.decode(q).float().cpu().numpy()
        for s in range(2):
            ref = o.decode_sequence(q[s].cpu().numpy().astype(np.float64), k_hat[s], v_hat[s], g)
            for hq in range(2 * g):
                assert rel_l2(out[s, hq], ref[hq]) <= ATTN_REL_L2_MAX


def test_decode_independent_of_split_count():
    # 40 tiles in sequence 0: 20 and 40 splits merge in two levels (groups of
    # 16 chunks, then the groups), the others in one
    w = synth.workload("tiny", num_seqs=2, lens=(64 * 40 + 7, 640), num_kv_heads=2, group_size=4)
    cfg, cache, rk, rv = _prefilled(w)
    q = synth.queries(w, device="cuda")
    outs = [cache.decode(q, num_splits=s).float().cpu().numpy() for s in (1, 2, 5, 13, 20, 40, 0)]
    for other in outs[1:]:
        assert rel_l2(other, outs[0]) <= 1e-4


def test_decode_edge_lengths():
    # empty sequence -> zeros; shorter than a tile -> tail only; exact tile multiple
    w = synth.workload("tiny", num_seqs=4, lens=(0, 5, 128, 64 * 3 + 63), num_kv_heads=1, group_size=2)
    cfg, cache, rk, rv = _prefilled(w)
    q = synth.queries(w, device="cuda")
    out = cache.decode(q).float().cpu().numpy()
    assert not out[0].any()
    rk_h, rv_h, q_h = rk.cpu().numpy(), rv.cpu().numpy(), q.cpu().numpy()
    starts = _starts(w.lens)
    for s in range(1, 4):
        L = w.lens[s]
        ref = oracle_decode_sequence(cfg, rk_h[starts[s]:starts[s] + L], rv_h[starts[s]:starts[s] + L], q_h[s])
        for hq in range(2):
            assert rel_l2(out[s, hq], ref[hq]) <= ATTN_REL_L2_MAX


@pytest.mark.parametrize("num_seqs", [300, 1100])
def test_decode_many_sequences(num_seqs):
    # the schedule's longest-first order (a sort over up to 1024 sequences)
    # and its block-wide scan of the units, past one warp and past one block
    # (1100 sequences: the order as given); lengths log-uniform with empty
    # and tail-only sequences; a seeded sample of sequences against fp64
    # attention over the GPU's own pages
    rng = np.random.default_rng(4242 + num_seqs)
    lens = np.floor(np.exp(rng.uniform(0.0, math.log(700.0), num_seqs))).astype(np.int64) - 1
    lens[:3] = (0, 31, 32)
    w = synth.workload("tiny", num_seqs=num_seqs, lens=tuple(int(x) for x in lens), num_kv_heads=1, group_size=2,
                       tile_tokens=32, bits_k=4, bits_v=2, iters=1)
    cfg, cache, _, _ = _prefilled(w)
    q = synth.queries(w, device="cuda")
    out = cache.decode(q)
    again = cache.decode(q, num_splits=1)
    torch.cuda.synchronize()
    assert cache.status() == 0
    out_h, q_h = out.float().cpu().numpy(), q.cpu().numpy()
    assert not out_h[0].any()
    sample = sorted(set([1, 2, num_seqs - 1] + list(rng.choice(num_seqs, 30, replace=False))))
    for s in sample:
        if lens[s] == 0:
            assert not out_h[s].any()
            continue
        ref = decode_over_gpu_pages(cfg, cache, s, int(lens[s]), q_h[s])
        for hq in range(w.num_q_heads):
            assert rel_l2(out_h[s, hq], ref[hq]) <= ATTN_REL_L2_MAX, (s, hq)
    assert rel_l2(again.float().cpu().numpy(), out_h) <= 1e-4


# ------------------------------------------------------------------- append

@pytest.mark.parametrize("t,chunks", [(64, [1] * 70), (128, [3, 100, 1, 130, 7]), (32, [33, 1, 64, 2])])
def test_append_equals_prefill(t, chunks):
    # tokens appended in chunks (tiles completing inside appends, several per
    # call) give pages bit-identical to quantizing the same tokens directly,
    # and the same tails
    l0 = 2 * t + 5
    total = l0 + sum(chunks)
    w = synth.workload("qwen3_32b_burst", num_seqs=2, lens=(l0, l0), num_kv_heads=2, group_size=4,
                       tile_tokens=t)
    cfg, a = make_cache(w, extra_tokens=total)
    _, b = make_cache(w, extra_tokens=total)
    rk = synth.kv_rows(w, "k", 2 * total, device="cuda")
    rv = synth.kv_rows(w, "v", 2 * total, device="cuda")
    seq_rows = lambda r, s, lo, hi: r[s * total + lo:s * total + hi]  # noqa: E731
    pk = torch.cat([seq_rows(rk, s, 0, l0) for s in range(2)])
    pv = torch.cat([seq_rows(rv, s, 0, l0) for s in range(2)])
    a.prefill(pk, pv, [l0, l0])
    pos = l0
    for c in chunks:
        nk = torch.cat([seq_rows(rk, s, pos, pos + c) for s in range(2)])
        nv = torch.cat([seq_rows(rv, s, pos, pos + c) for s in range(2)])
        a.append(nk, nv, [c, c])
        pos += c
    b.prefill(rk, rv, [total, total])
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    bt = a.block_tables.cpu().numpy()
    full_blocks = (total // t) * (t // 16)
    used = bt[:, :full_blocks].ravel()
    assert torch.equal(a.k_pool[used], b.k_pool[used])
    assert torch.equal(a.v_pool[used], b.v_pool[used])
    tau = total % t
    assert torch.equal(a.k_tail[:, :, :tau], b.k_tail[:, :, :tau])
    assert torch.equal(a.v_tail[:, :, :tau], b.v_tail[:, :, :tau])
    q = synth.queries(w, device="cuda")
    assert torch.equal(a.decode(q), b.decode(q))
