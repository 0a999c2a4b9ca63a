"""Head sizes d = 64 and 256 (the method's rotation along the head-dim
channels of any head size: axbrief.com KVarN article, "What differs from
existing methods"): quantize, append, decode and chunked prefill through the
C ABI against the oracle, with the same bars as the d = 128 tests."""

import numpy as np
import pytest
import torch

from oracle import kvq_oracle as o
from quantized_paged_kv_tile_b200 import kvq, synth
from quantized_paged_kv_tile_b200.paged import PagedKVCache

from parity_helpers import (ATTN_REL_L2_MAX, TileStats, compare_sequence_tiles, decode_over_gpu_pages,
                            gpu_pages_kv_hat, make_cache, rel_l2)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kvq.load_library()


def _starts(lens):
    return np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)


def _prefilled(w, num_splits=0, extra_tokens=0, rotation_seed=0):
    if rotation_seed:
        cfg = kvq.Config(num_kv_heads=w.num_kv_heads, group_size=w.group_size, tile_tokens=w.tile_tokens,
                         bits_k=w.bits_k, bits_v=w.bits_v, iters=w.iters, head_dim=w.head_dim,
                         rotation_seed=rotation_seed)
        bps = -(-(max(w.lens) + extra_tokens) // 16)
        cache = PagedKVCache(cfg, w.num_seqs, bps * 16, block_table=synth.block_table(w, bps), num_splits=num_splits)
    else:
        cfg, cache = make_cache(w, extra_tokens=extra_tokens, num_splits=num_splits)
    total = int(sum(w.lens))
    rk = synth.kv_rows(w, "k", total, device="cuda")
    rv = synth.kv_rows(w, "v", total, device="cuda")
    cache.prefill(rk, rv, w.lens)
    torch.cuda.synchronize()
    assert cache.status() == 0
    return cfg, cache, rk, rv


QUANT_CASES = [
    # (d, T, bits_k, bits_v, iters, heads, lens, rotation seed)
    (64, 64, 4, 4, 4, 2, (300, 129), 0),
    (64, 32, 2, 3, 1, 1, (200, 96), 0),
    (64, 128, 8, 8, 2, 1, (260,), 0),
    (64, 64, 4, 2, 8, 1, (192,), 0x9E37),   # randomized rotation
    (256, 64, 4, 4, 4, 2, (200, 70), 0),
    (256, 128, 3, 4, 2, 1, (300,), 0),
    (256, 32, 2, 2, 0, 1, (100,), 0),       # n = 0
    (256, 64, 8, 8, 1, 1, (130,), 0x51),    # 8-bit codes, randomized rotation
]


@pytest.mark.parametrize("d,t,bk,bv,n,h,lens,seed", QUANT_CASES)
def test_quantize_matches_oracle(d, t, bk, bv, n, h, lens, seed):
    w = synth.workload("prefill_sweep", num_seqs=len(lens), lens=lens, num_kv_heads=h, tile_tokens=t,
                       bits_k=bk, bits_v=bv, iters=n, head_dim=d)
    cfg, cache, rk, rv = _prefilled(w, rotation_seed=seed)
    rk_h, rv_h = rk.cpu().numpy(), rv.cpu().numpy()
    tiles = [(s, i) for s in range(len(lens)) for i in range(lens[s] // t)]
    sk, sv = TileStats(), TileStats()
    compare_sequence_tiles(cfg, cache, rk_h, rv_h, _starts(lens), tiles, sk, sv)
    sk.check()
    sv.check()
    kt, vt = cache.k_tail.cpu().numpy(), cache.v_tail.cpu().numpy()
    for s, L in enumerate(lens):
        tau = L % t
        r0 = _starts(lens)[s] + L - tau
        for hh in range(h):
            np.testing.assert_array_equal(kt[s, hh, :tau], rk_h[r0:r0 + tau, hh])
            np.testing.assert_array_equal(vt[s, hh, :tau], rv_h[r0:r0 + tau, hh])


@pytest.mark.parametrize("d,t,chunks", [(64, 32, [1] * 40), (256, 64, [3, 100, 1, 70]), (64, 128, [130, 7, 1])])
def test_append_equals_prefill(d, t, chunks):
    # tokens appended in chunks (tiles completing inside appends, several per
    # call) give pages bit-identical to quantizing the same tokens directly
    l0 = 2 * t + 5
    total = l0 + sum(chunks)
    w = synth.workload("qwen3_32b_burst", num_seqs=2, lens=(l0, l0), num_kv_heads=2, group_size=4,
                       tile_tokens=t, head_dim=d)
    cfg, a = make_cache(w, extra_tokens=total)
    _, b = make_cache(w, extra_tokens=total)
    rk = synth.kv_rows(w, "k", 2 * total, device="cuda")
    rv = synth.kv_rows(w, "v", 2 * total, device="cuda")
    seq_rows = lambda r, s, lo, hi: r[s * total + lo:s * total + hi]  # noqa: E731
    a.prefill(torch.cat([seq_rows(rk, s, 0, l0) for s in range(2)]),
              torch.cat([seq_rows(rv, s, 0, l0) for s in range(2)]), [l0, l0])
    pos = l0
    for c in chunks:
        a.append(torch.cat([seq_rows(rk, s, pos, pos + c) for s in range(2)]),
                 torch.cat([seq_rows(rv, s, pos, pos + c) for s in range(2)]), [c, c])
        pos += c
    b.prefill(rk, rv, [total, total])
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    bt = a.block_tables.cpu().numpy()
    used = bt[:, :(total // t) * (t // 16)].ravel()
    assert torch.equal(a.k_pool[used], b.k_pool[used])
    assert torch.equal(a.v_pool[used], b.v_pool[used])
    tau = total % t
    assert torch.equal(a.k_tail[:, :, :tau], b.k_tail[:, :, :tau])
    assert torch.equal(a.v_tail[:, :, :tau], b.v_tail[:, :, :tau])
    q = synth.queries(w, device="cuda")
    assert torch.equal(a.decode(q), b.decode(q))


DECODE_CASES = [
    # (d, T, bits_k, bits_v, g, lens, splits)
    (64, 64, 4, 4, 4, (3 * 64 + 9, 64 * 5), 0),
    (64, 32, 2, 3, 8, (7 * 32 + 31,), 3),
    (64, 128, 8, 8, 2, (2 * 128 + 1, 50), 1),
    (256, 64, 4, 2, 8, (4 * 64 + 17, 3 * 64), 0),
    (256, 128, 3, 3, 4, (3 * 128 + 127,), 2),
    (256, 32, 4, 4, 1, (9 * 32 + 5, 31, 0), 4),
]


@pytest.mark.parametrize("d,t,bk,bv,g,lens,splits", DECODE_CASES)
def test_decode_matches_oracle(d, t, bk, bv, g, lens, splits):
    # decode over the cache is held to 1e-3 against fp64 attention over the
    # GPU's own pages (read by the oracle) and raw tail; the pages themselves
    # are held to the quantize bars above (every differing code a rounding tie)
    w = synth.workload("tiny", num_seqs=len(lens), lens=lens, num_kv_heads=2, group_size=g, tile_tokens=t,
                       bits_k=bk, bits_v=bv, iters=2, head_dim=d)
    cfg, cache, rk, rv = _prefilled(w, num_splits=splits)
    q = synth.queries(w, device="cuda")
    out = cache.decode(q)
    torch.cuda.synchronize()
    assert cache.status() == 0
    out_h, q_h = out.float().cpu().numpy(), q.cpu().numpy()
    for s, L in enumerate(lens):
        if L == 0:
            assert not out_h[s].any()
            continue
        ref = decode_over_gpu_pages(cfg, cache, s, L, q_h[s])
        for hq in range(w.num_q_heads):
            assert rel_l2(out_h[s, hq], ref[hq]) <= ATTN_REL_L2_MAX, (s, hq)
    tiles = [(s, i) for s in range(len(lens)) for i in range(lens[s] // t)]
    sk, sv = TileStats(), TileStats()
    compare_sequence_tiles(cfg, cache, rk.cpu().numpy(), rv.cpu().numpy(), _starts(lens), tiles, sk, sv)
    sk.check()
    sv.check()


@pytest.mark.parametrize("d", [64, 256])
def test_decode_independent_of_split_count(d):
    w = synth.workload("tiny", num_seqs=2, lens=(64 * 20 + 7, 300), num_kv_heads=2, group_size=4, head_dim=d)
    cfg, cache, rk, rv = _prefilled(w)
    q = synth.queries(w, device="cuda")
    outs = [cache.decode(q, num_splits=s).float().cpu().numpy() for s in (1, 2, 7, 20, 0)]
    for other in outs[1:]:
        assert rel_l2(other, outs[0]) <= 1e-4


PREFILL_CASES = [
    # (d, T, bits_k, bits_v, g, context lengths, chunk lengths)
    (64, 64, 4, 4, 4, (300, 64, 0), (40, 33, 17)),   # ragged tails, a tail-free context, an empty context
    (64, 32, 2, 3, 8, (100, 31), (20, 1)),           # 3-bit V, a context that is all tail
    (64, 128, 8, 8, 1, (260,), (70,)),               # g = 1: 32 chunk tokens per CTA, three runs
    (256, 64, 4, 2, 8, (200, 70), (9, 30)),          # 2 chunk tokens per CTA
    (256, 128, 3, 4, 2, (300,), (25,)),
    (256, 32, 2, 2, 4, (97, 64), (0, 40)),           # a sequence with an empty chunk
]


@pytest.mark.parametrize("d,t,bk,bv,g,ctx,chunk", PREFILL_CASES)
def test_prefill_attention_matches_oracle(d, t, bk, bv, g, ctx, chunk):
    # chunk token i attends to the cached context (the GPU's own pages, read
    # back by the oracle, then the raw tail) and to chunk rows 0..i: fp64
    # attention held to 1e-3 per (chunk token, query head); the result does
    # not depend on the split count (the context is not split at these sizes)
    w = synth.workload("tiny", num_seqs=len(ctx), lens=tuple(ctx), num_kv_heads=2, group_size=g, tile_tokens=t,
                       bits_k=bk, bits_v=bv, iters=2, head_dim=d)
    cfg, cache, _, _ = _prefilled(w, extra_tokens=max(chunk))
    n = int(sum(chunk))
    k_new = synth.kv_rows(w, "k", max(n, 1), device="cuda", stream_id=3)[:n]
    v_new = synth.kv_rows(w, "v", max(n, 1), device="cuda", stream_id=3)[:n]
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7100 + d)
    q = torch.randn((n, w.num_q_heads, d), generator=gen, device="cuda").to(torch.float16)
    out = cache.prefill_chunk(q, k_new, v_new, chunk, append=False)
    again = cache.prefill_chunk(q, k_new, v_new, chunk, append=False, num_splits=5)
    torch.cuda.synchronize()
    assert cache.status() == 0
    assert torch.equal(out, again)
    qh, kh, vh, oh = (x.float().cpu().numpy() for x in (q, k_new, v_new, out))
    assert np.all(np.isfinite(oh))
    starts = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int64)
    for s, c in enumerate(chunk):
        if c == 0:
            continue
        k_hat = [gpu_pages_kv_hat(cfg, cache, s, h, int(ctx[s]), False) for h in range(cfg.num_kv_heads)]
        v_hat = [gpu_pages_kv_hat(cfg, cache, s, h, int(ctx[s]), True) for h in range(cfg.num_kv_heads)]
        a, b = starts[s], starts[s] + c
        ref = o.prefill_chunk_sequence(qh[a:b], k_hat, v_hat, kh[a:b], vh[a:b], cfg.group_size)
        for i in range(c):
            for hq in range(cfg.num_q_heads):
                assert rel_l2(oh[a + i, hq], ref[i, hq]) <= ATTN_REL_L2_MAX, (s, i, hq)


@pytest.mark.parametrize("d", [64, 256])
def test_prefill_chunk_then_append_matches_one_prefill(d):
    # attention, then the chunk joins the cache (tiles it completes are
    # quantized): pages and tails equal to one prefill of context + chunk
    ctx, chunk = (130, 64, 5), (70, 1, 200)
    w = synth.workload("tiny", num_seqs=3, lens=ctx, num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=4,
                       bits_v=2, iters=2, head_dim=d)
    cfg, a, _, _ = _prefilled(w, extra_tokens=max(chunk))
    n = int(sum(chunk))
    k_new = synth.kv_rows(w, "k", n, device="cuda", stream_id=4)
    v_new = synth.kv_rows(w, "v", n, device="cuda", stream_id=4)
    q = torch.zeros((n, w.num_q_heads, d), dtype=torch.float16, device="cuda")
    a.prefill_chunk(q, k_new, v_new, chunk)
    rk = synth.kv_rows(w, "k", int(sum(ctx)), device="cuda")
    rv = synth.kv_rows(w, "v", int(sum(ctx)), device="cuda")
    cs, ns = np.concatenate([[0], np.cumsum(ctx)]), np.concatenate([[0], np.cumsum(chunk)])
    full_k = torch.cat([torch.cat([rk[cs[s]:cs[s + 1]], k_new[ns[s]:ns[s + 1]]]) for s in range(3)])
    full_v = torch.cat([torch.cat([rv[cs[s]:cs[s + 1]], v_new[ns[s]:ns[s + 1]]]) for s in range(3)])
    totals = [c + m for c, m in zip(ctx, chunk)]
    _, b = make_cache(w, extra_tokens=max(chunk))
    b.prefill(full_k, full_v, totals)
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    for s, L in enumerate(totals):
        used = a.block_tables[s, :(L // 64) * 4].long()
        assert torch.equal(a.k_pool[used], b.k_pool[used]) and torch.equal(a.v_pool[used], b.v_pool[used])
        assert torch.equal(a.k_tail[s, :, :L % 64], b.k_tail[s, :, :L % 64])
        assert torch.equal(a.v_tail[s, :, :L % 64], b.v_tail[s, :, :L % 64])


def _chunk_setup(d, ctx, chunk, g=4, t=64):
    w = synth.workload("tiny", num_seqs=len(ctx), lens=tuple(ctx), num_kv_heads=2, group_size=g, tile_tokens=t,
                       bits_k=4, bits_v=4, iters=2, head_dim=d)
    cfg, cache, _, _ = _prefilled(w, extra_tokens=max(chunk))
    n = int(sum(chunk))
    k_new = synth.kv_rows(w, "k", n, device="cuda", stream_id=5)
    v_new = synth.kv_rows(w, "v", n, device="cuda", stream_id=5)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(7300 + d)
    q = torch.randn((n, w.num_q_heads, d), generator=gen, device="cuda").to(torch.float16)
    return w, cfg, cache, q, k_new, v_new


@pytest.mark.parametrize("d", [64, 256])
def test_one_token_chunk_matches_decode_after_append(d):
    # both GPU paths at this head size: a one-token chunk (the token raw)
    # against appending it and decoding (the token in the tail, raw too)
    w, cfg, cache, q, k_new, v_new = _chunk_setup(d, (300, 70, 129), (1, 1, 1))  # no tile completes
    out = cache.prefill_chunk(q, k_new, v_new, (1, 1, 1), append=True)
    dec = cache.decode(q)
    torch.cuda.synchronize()
    assert cache.status() == 0
    a, b = out.float().cpu().numpy(), dec.float().cpu().numpy()
    for s in range(3):
        for hq in range(w.num_q_heads):
            assert rel_l2(a[s, hq], b[s, hq]) <= ATTN_REL_L2_MAX


@pytest.mark.parametrize("d", [64, 256])
def test_prefill_chunk_longer_than_bound_is_reported(d):
    w, cfg, cache, q, k_new, v_new = _chunk_setup(d, (200, 90), (10, 12))
    cu = torch.tensor([0, 10, 22], dtype=torch.int32, device="cuda")
    out = torch.full_like(q, float("nan"))
    kvq.paged_prefill_attention(cfg, q, out, k_new, v_new, cu, cache.seq_lens, 11, cache.block_tables,
                                cache.k_pool, cache.v_pool, cache.k_tail, cache.v_tail,
                                num_blocks=cache.num_blocks, dev_status=cache.dev_status)
    torch.cuda.synchronize()
    assert cache.status() == kvq.KVQ_ERR_DEVICE_BOUNDS
    oh = out.float().cpu().numpy()
    assert np.all(np.isfinite(oh[:21])) and np.all(np.isnan(oh[21]))  # rows past the bound untouched
    cache.dev_status.zero_()
    full = cache.prefill_chunk(q, k_new, v_new, (10, 12), append=False)
    torch.cuda.synchronize()
    assert torch.equal(full[:21], out[:21])


@pytest.mark.parametrize("d", [64, 256])
def test_prefill_tile_outside_pool_is_skipped_and_reported(d):
    # one tile of sequence 0 points outside the pool: reported, and the
    # output is attention over the context without that tile's tokens
    ctx, chunk = (640, 300), (24, 40)
    w, cfg, cache, q, k_new, v_new = _chunk_setup(d, ctx, chunk)
    k_hat = [gpu_pages_kv_hat(cfg, cache, 0, h, ctx[0], False) for h in range(cfg.num_kv_heads)]
    v_hat = [gpu_pages_kv_hat(cfg, cache, 0, h, ctx[0], True) for h in range(cfg.num_kv_heads)]
    bad_tile, t, per = 3, cfg.tile_tokens, cfg.tile_tokens // cfg.page_tokens
    cache.block_tables[0, bad_tile * per + 1] = cache.num_blocks + 7
    out = cache.prefill_chunk(q, k_new, v_new, chunk, append=False)
    torch.cuda.synchronize()
    assert cache.status() == kvq.KVQ_ERR_DEVICE_BOUNDS
    keep = np.r_[0:bad_tile * t, (bad_tile + 1) * t:ctx[0]]
    qh, kh, vh, oh = (x.float().cpu().numpy() for x in (q, k_new, v_new, out))
    ref = o.prefill_chunk_sequence(qh[:24], [k[keep] for k in k_hat], [v[keep] for v in v_hat], kh[:24], vh[:24],
                                   cfg.group_size)
    for i in range(24):
        for hq in range(cfg.num_q_heads):
            assert rel_l2(oh[i, hq], ref[i, hq]) <= ATTN_REL_L2_MAX
    assert np.all(np.isfinite(oh))


@pytest.mark.parametrize("d", [64, 256])
def test_serving_step_equals_append_then_decode(d):
    # the serving step at this head size (tail write and length update, then
    # the decode) against kvq_append_tokens, the lengths advanced, and
    # kvq_paged_decode_attention with the same split count: identical outputs,
    # tails and lengths, step after step
    w = synth.workload("tiny", num_seqs=2, lens=(64 * 9 + 3, 64 * 4 + 9), num_kv_heads=2, group_size=4,
                       head_dim=d)
    cfg, a, _, _ = _prefilled(w, extra_tokens=8)
    _, b, _, _ = _prefilled(w, extra_tokens=8)
    ws = torch.zeros(kvq.decode_workspace_bytes(cfg, 2, 3), dtype=torch.uint8, device="cuda")
    for i in range(8):
        nk = synth.kv_rows(w, "k", 2, device="cuda", stream_id=1 + i)
        nv = synth.kv_rows(w, "v", 2, device="cuda", stream_id=1 + i)
        q = synth.queries(w, device="cuda", step=i)
        a.append(nk, nv)
        out_a = a.decode(q, num_splits=3)
        out_b = torch.empty_like(q)
        kvq.append_decode_step(cfg, nk, nv, q, out_b, b.seq_lens, b.block_tables, b.k_pool, b.v_pool, b.k_tail,
                               b.v_tail, ws, 3, num_blocks=b.num_blocks, dev_status=b.dev_status)
        assert torch.equal(out_a, out_b), i
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    assert torch.equal(a.seq_lens, b.seq_lens)
    assert torch.equal(a.k_tail, b.k_tail) and torch.equal(a.v_tail, b.v_tail)


@pytest.mark.parametrize("d", [64, 256])
def test_serving_step_refuses_a_tile_completion(d):
    w = synth.workload("tiny", num_seqs=2, lens=(63, 40), num_kv_heads=1, group_size=2, head_dim=d)
    cfg, c, _, _ = _prefilled(w, extra_tokens=2)
    ws = torch.zeros(kvq.decode_workspace_bytes(cfg, 2, 2), dtype=torch.uint8, device="cuda")
    nk = torch.ones((2, 1, d), dtype=torch.float16, device="cuda")
    q = synth.queries(w, device="cuda")
    out = torch.empty_like(q)
    tail_before = c.k_tail.clone()
    kvq.append_decode_step(cfg, nk, nk, q, out, c.seq_lens, c.block_tables, c.k_pool, c.v_pool, c.k_tail, c.v_tail,
                           ws, 2, num_blocks=c.num_blocks, dev_status=c.dev_status)
    torch.cuda.synchronize()
    assert c.status() == kvq.KVQ_ERR_DEVICE_BOUNDS
    assert torch.equal(c.k_tail[0], tail_before[0])      # sequence 0 (63 -> 64) not written
    assert torch.equal(c.k_tail[1, 0, 40], nk[1, 0])     # sequence 1 appended at row 40
    assert c.seq_lens.tolist() == [64, 41]
