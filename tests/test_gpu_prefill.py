"""GPU parity of chunked prefill attention over the quantized cache
(kvq_paged_prefill_attention) against the oracle's prefill_chunk_sequence.

The oracle reads the context from the GPU's own pages (decoded by the
oracle's page reader), so these tests isolate the read path; the write
path's pages are held to the quantize bars by the other parity tests.
Tolerance: relative L2 <= 1e-3 per (chunk token, query head).
"""

import numpy as np
import pytest
import torch

from oracle import kvq_oracle as o
from quantized_paged_kv_tile_b200 import kvq, synth

from parity_helpers import ATTN_REL_L2_MAX, gpu_pages_kv_hat, make_cache, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    kvq.load_library()


def _chunk_inputs(w, counts, seed):
    n = int(sum(counts))
    k_new = synth.kv_rows(w, "k", n, device="cuda", stream_id=seed)
    v_new = synth.kv_rows(w, "v", n, device="cuda", stream_id=seed)
    g = torch.Generator(device="cuda")
    g.manual_seed(7000 + seed)
    q = torch.randn((n, w.num_q_heads, 128), generator=g, device="cuda").to(torch.float16)
    return q, k_new, v_new


def _setup(t, bk, bv, g, ctx, chunk, rotation_seed=0, seed=1):
    w = synth.workload("tiny", num_seqs=len(ctx), lens=tuple(ctx), num_kv_heads=2, group_size=g, tile_tokens=t,
                       bits_k=bk, bits_v=bv, iters=2)
    cfg0, cache = make_cache(w, extra_tokens=max(chunk))
    if rotation_seed:
        from quantized_paged_kv_tile_b200.paged import PagedKVCache
        cfg = kvq.Config(num_kv_heads=2, group_size=g, tile_tokens=t, bits_k=bk, bits_v=bv, iters=2,
                         rotation_seed=rotation_seed)
        bps = cache.blocks_per_seq
        cache = PagedKVCache(cfg, w.num_seqs, bps * 16, block_table=synth.block_table(w, bps))
    total = int(sum(ctx))
    rk = synth.kv_rows(w, "k", max(total, 1), device="cuda")[:total]
    rv = synth.kv_rows(w, "v", max(total, 1), device="cuda")[:total]
    cache.prefill(rk, rv, ctx)
    q, k_new, v_new = _chunk_inputs(w, chunk, seed)
    return w, cache, q, k_new, v_new


def _check_against_oracle(w, cache, ctx, chunk, q, k_new, v_new, out):
    cfg = cache.cfg
    qh, kh, vh, oh = (x.float().cpu().numpy() for x in (q, k_new, v_new, out))
    assert np.all(np.isfinite(oh))
    starts = np.concatenate([[0], np.cumsum(chunk)]).astype(np.int64)
    worst = 0.0
    for s in range(len(ctx)):
        n = int(chunk[s])
        if n == 0:
            continue
        k_hat = [gpu_pages_kv_hat(cfg, cache, s, h, int(ctx[s]), False) for h in range(cfg.num_kv_heads)]
        v_hat = [gpu_pages_kv_hat(cfg, cache, s, h, int(ctx[s]), True) for h in range(cfg.num_kv_heads)]
        a, b = starts[s], starts[s] + n
        ref = o.prefill_chunk_sequence(qh[a:b], k_hat, v_hat, kh[a:b], vh[a:b], cfg.group_size)
        for i in range(n):
            for hq in range(cfg.num_q_heads):
                err = rel_l2(oh[a + i, hq], ref[i, hq])
                worst = max(worst, err)
                assert err <= ATTN_REL_L2_MAX, (s, i, hq, err)
    return worst


CASES = [
    # (T, bits_k, bits_v, g, context lengths, chunk lengths)
    (64, 4, 4, 4, (700, 64, 0), (40, 33, 17)),     # ragged tails, empty context, two 128-row tiles
    (32, 4, 2, 8, (300, 31), (20, 1)),              # T = 32 (half-empty MMA blocks), context all tail
    (128, 2, 4, 2, (1000, 129), (70, 5)),           # two MMA blocks per tile
    (64, 8, 8, 1, (400,), (130,)),                  # g = 1, 8-bit codes
    (128, 8, 8, 4, (256, 300), (9, 50)),
    (64, 2, 2, 4, (513, 77), (64, 0)),              # a sequence with an empty chunk
    (32, 8, 8, 2, (100, 0), (64, 3)),
    (64, 3, 3, 4, (300, 70), (40, 17)),             # 3-bit codes (token-major bitstreams)
    (128, 3, 4, 2, (260,), (30,)),
    (32, 4, 3, 8, (97, 64), (21, 40)),
]


@pytest.mark.parametrize("t,bk,bv,g,ctx,chunk", CASES)
def test_prefill_attention_matches_oracle(t, bk, bv, g, ctx, chunk):
    w, cache, q, k_new, v_new = _setup(t, bk, bv, g, ctx, chunk)
    out = cache.prefill_chunk(q, k_new, v_new, chunk, append=False)
    torch.cuda.synchronize()
    assert cache.status() == 0
    _check_against_oracle(w, cache, ctx, chunk, q, k_new, v_new, out)


@pytest.mark.parametrize("splits", [2, 3, 7])
@pytest.mark.parametrize("t,bk,bv,g,ctx,chunk", [CASES[0], CASES[1], CASES[2], CASES[4]])
def test_prefill_attention_context_splits(t, bk, bv, g, ctx, chunk, splits):
    # the context tiles split over several CTAs (some splits empty when a
    # context has fewer tiles than splits), merged by a second launch
    w, cache, q, k_new, v_new = _setup(t, bk, bv, g, ctx, chunk)
    out = cache.prefill_chunk(q, k_new, v_new, chunk, append=False, num_splits=splits)
    one = cache.prefill_chunk(q, k_new, v_new, chunk, append=False, num_splits=1)
    torch.cuda.synchronize()
    assert cache.status() == 0
    _check_against_oracle(w, cache, ctx, chunk, q, k_new, v_new, out)
    # split and unsplit agree to fp32 rounding before the fp16 output; two
    # fp16 roundings of such values differ by at most one ulp, <= 2^-10 relative
    oh, uh = out.float().cpu().numpy(), one.float().cpu().numpy()
    assert max(rel_l2(oh[i, j], uh[i, j]) for i in range(oh.shape[0]) for j in range(oh.shape[1])) <= 2.0 ** -10


def test_prefill_attention_randomized_rotation():
    ctx, chunk = (513, 200), (64, 31)
    w, cache, q, k_new, v_new = _setup(64, 4, 4, 4, ctx, chunk, rotation_seed=1234567)
    out = cache.prefill_chunk(q, k_new, v_new, chunk, append=False)
    torch.cuda.synchronize()
    assert cache.status() == 0
    _check_against_oracle(w, cache, ctx, chunk, q, k_new, v_new, out)


def test_prefill_chunk_appends_like_prefill():
    # attention, then the chunk joins the cache: pages and tails equal to a
    # cache that was prefilled with context + chunk in one go
    ctx, chunk = (130, 64, 5), (70, 1, 200)
    w, cache, q, k_new, v_new = _setup(64, 4, 2, 4, ctx, chunk)
    cache.prefill_chunk(q, k_new, v_new, chunk)
    torch.cuda.synchronize()
    assert cache.status() == 0
    assert list(cache.host_lens) == [c + n for c, n in zip(ctx, chunk)]
    assert cache.seq_lens.cpu().tolist() == list(cache.host_lens)
    # the same rows, packed per sequence, into a fresh cache
    total = int(sum(ctx))
    rk = synth.kv_rows(w, "k", total, device="cuda")
    rv = synth.kv_rows(w, "v", total, device="cuda")
    cs, ns = np.concatenate([[0], np.cumsum(ctx)]), np.concatenate([[0], np.cumsum(chunk)])
    pk = torch.cat([torch.cat([rk[cs[s]:cs[s + 1]], k_new[ns[s]:ns[s + 1]]]) for s in range(len(ctx))])
    pv = torch.cat([torch.cat([rv[cs[s]:cs[s + 1]], v_new[ns[s]:ns[s + 1]]]) for s in range(len(ctx))])
    lens = [c + n for c, n in zip(ctx, chunk)]
    _, fresh = make_cache(w, extra_tokens=max(chunk))
    fresh.prefill(pk, pv, lens)
    torch.cuda.synchronize()
    assert torch.equal(cache.k_pool, fresh.k_pool) and torch.equal(cache.v_pool, fresh.v_pool)
    t = cache.cfg.tile_tokens
    for s, n in enumerate(lens):
        tau = n % t
        assert torch.equal(cache.k_tail[s, :, :tau], fresh.k_tail[s, :, :tau])
        assert torch.equal(cache.v_tail[s, :, :tau], fresh.v_tail[s, :, :tau])


def test_one_token_chunk_matches_decode_after_append():
    # both GPU paths: a one-token chunk (token raw) against appending it and
    # decoding (token in the tail, raw too: no tile completes)
    ctx = (300, 70, 129)
    w, cache, q, k_new, v_new = _setup(64, 4, 4, 4, ctx, (1, 1, 1))
    out = cache.prefill_chunk(q, k_new, v_new, (1, 1, 1), append=True)
    dec = cache.decode(q)
    torch.cuda.synchronize()
    assert cache.status() == 0
    a, b = out.float().cpu().numpy(), dec.float().cpu().numpy()
    for s in range(3):
        for hq in range(w.num_q_heads):
            assert rel_l2(a[s, hq], b[s, hq]) <= ATTN_REL_L2_MAX


def test_prefill_chunk_longer_than_bound_is_reported():
    ctx, chunk = (200, 90), (10, 12)
    w, cache, q, k_new, v_new = _setup(64, 4, 4, 4, ctx, chunk)
    cu = torch.tensor([0, 10, 22], dtype=torch.int32, device="cuda")
    out = torch.full_like(q, float("nan"))
    kvq.paged_prefill_attention(cache.cfg, q, out, k_new, v_new, cu, cache.seq_lens, 11, cache.block_tables,
                                cache.k_pool, cache.v_pool, cache.k_tail, cache.v_tail,
                                num_blocks=cache.num_blocks, dev_status=cache.dev_status)
    torch.cuda.synchronize()
    assert cache.status() == kvq.KVQ_ERR_DEVICE_BOUNDS
    oh = out.float().cpu().numpy()
    assert np.all(np.isfinite(oh[:21])) and np.all(np.isnan(oh[21]))   # rows past the bound untouched
    cache.dev_status.zero_()
    # the rows within the bound are still right
    full = cache.prefill_chunk(q, k_new, v_new, chunk, append=False)
    torch.cuda.synchronize()
    fh = full.float().cpu().numpy()
    for r in range(21):
        for hq in range(w.num_q_heads):
            assert rel_l2(oh[r, hq], fh[r, hq]) <= 1e-6


def test_prefill_tile_outside_pool_is_skipped_and_reported():
    # one tile of sequence 0 points outside the pool: reported, and the
    # output is attention over the context without that tile's tokens
    ctx, chunk = (640, 300), (24, 40)
    w, cache, q, k_new, v_new = _setup(64, 4, 4, 4, ctx, chunk)
    cfg = cache.cfg
    k_hat = [gpu_pages_kv_hat(cfg, cache, 0, h, ctx[0], False) for h in range(cfg.num_kv_heads)]
    v_hat = [gpu_pages_kv_hat(cfg, cache, 0, h, ctx[0], True) for h in range(cfg.num_kv_heads)]
    bad_tile, t, per = 3, cfg.tile_tokens, cfg.tile_tokens // cfg.page_tokens
    cache.block_tables[0, bad_tile * per + 1] = cache.num_blocks + 7
    out = cache.prefill_chunk(q, k_new, v_new, chunk, append=False, num_splits=2)
    torch.cuda.synchronize()
    assert cache.status() == kvq.KVQ_ERR_DEVICE_BOUNDS
    keep = np.r_[0:bad_tile * t, (bad_tile + 1) * t:ctx[0]]
    k_cut = [k[keep] for k in k_hat]
    v_cut = [v[keep] for v in v_hat]
    qh, kh, vh, oh = (x.float().cpu().numpy() for x in (q, k_new, v_new, out))
    ref = o.prefill_chunk_sequence(qh[:24], k_cut, v_cut, kh[:24], vh[:24], cfg.group_size)
    for i in range(24):
        for hq in range(cfg.num_q_heads):
            assert rel_l2(oh[i, hq], ref[i, hq]) <= ATTN_REL_L2_MAX
    assert np.all(np.isfinite(oh))
