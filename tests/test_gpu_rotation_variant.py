"""GPU parity of the randomized-rotation variant (kvq_config.rotation_seed
!= 0: X' = X D_s H with SplitMix64 channel signs) against the oracle's
variant, through the C ABI: quantized pages, the original-domain read-back,
end-to-end decode, and appends equal to prefill."""

import dataclasses

import numpy as np
import pytest
import torch

from oracle import kvq_oracle as o
from quantized_paged_kv_tile_b200 import kvq, synth
from quantized_paged_kv_tile_b200.paged import PagedKVCache

from parity_helpers import ATTN_REL_L2_MAX, TileStats, rel_l2, unpack_all

pytestmark = pytest.mark.gpu

SEED = 0x9E3779B9


def _cache(w, seed, extra_tokens=0, num_splits=0):
    cfg = kvq.Config(num_kv_heads=w.num_kv_heads, group_size=w.group_size, tile_tokens=w.tile_tokens,
                     bits_k=w.bits_k, bits_v=w.bits_v, iters=w.iters, rotation_seed=seed)
    max_tokens = max(w.lens) + max(extra_tokens, w.append_tokens)
    bps = -(-max(max_tokens, 1) // 16)
    return cfg, PagedKVCache(cfg, w.num_seqs, bps * 16, block_table=synth.block_table(w, bps), num_splits=num_splits)


def _starts(lens):
    return np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)


@pytest.mark.parametrize("t,bk,bv,n", [(64, 4, 2, 4), (128, 3, 4, 2), (32, 2, 2, 1)])
def test_seeded_quantize_matches_oracle(t, bk, bv, n):
    w = synth.workload("prefill_sweep", num_seqs=2, lens=(3 * t + 17, 2 * t), num_kv_heads=2, tile_tokens=t,
                       bits_k=bk, bits_v=bv, iters=n)
    cfg, cache = _cache(w, SEED)
    total = int(sum(w.lens))
    rk = synth.kv_rows(w, "k", total, device="cuda")
    rv = synth.kv_rows(w, "v", total, device="cuda")
    cache.prefill(rk, rv, w.lens)
    torch.cuda.synchronize()
    assert cache.status() == 0
    rk_h, rv_h = rk.cpu().numpy(), rv.cpu().numpy()
    starts = _starts(w.lens)
    tiles = [(s, i) for s in range(2) for i in range(w.lens[s] // t)]
    sk, sv = TileStats(), TileStats()
    for rows, is_v, bits, st in ((rk_h, False, bk, sk), (rv_h, True, bv, sv)):
        g = unpack_all(cfg, cache, tiles, is_v)
        for j, (s, i) in enumerate(tiles):
            for h in range(2):
                x = rows[starts[s] + i * t:starts[s] + (i + 1) * t, h]
                ref = o.quantize_tile(x, bits, n, dtype=np.float32, seed=SEED)
                st.add(g["codes"][j, h], g["meta"][j, h], g["cvec"][j, h], g["rot"][j, h], ref,
                       src=(x, bits, n, SEED))
                # the GPU's original-domain read-back applies H D_s
                _, ref_orig = o.dequantize_tile(g["codes"][j, h], g["meta"][j, h][:, 0], g["meta"][j, h][:, 1],
                                                g["cvec"][j, h], SEED)
                np.testing.assert_allclose(g["orig"][j, h], ref_orig, rtol=1e-4,
                                           atol=1e-5 * max(np.abs(ref_orig).max(), 1e-6))
    sk.check()
    sv.check()


def test_seeded_decode_matches_oracle():
    w = synth.workload("tiny", num_seqs=3, lens=(700, 64, 30), num_kv_heads=2, group_size=4, bits_v=2)
    cfg, cache = _cache(w, SEED)
    total = int(sum(w.lens))
    rk = synth.kv_rows(w, "k", total, device="cuda")
    rv = synth.kv_rows(w, "v", total, device="cuda")
    cache.prefill(rk, rv, w.lens)
    q = synth.queries(w, device="cuda")
    out = cache.decode(q)
    # the same pages read with the plain rotation give a different output
    plain = dataclasses.replace(cfg, rotation_seed=0)
    out_plain = torch.empty_like(q)
    kvq.paged_decode_attention(plain, q, out_plain, cache.seq_lens, cache.block_tables, cache.k_pool, cache.v_pool,
                               cache.k_tail, cache.v_tail, cache.workspace, num_blocks=cache.num_blocks)
    torch.cuda.synchronize()
    assert cache.status() == 0
    rk_h, rv_h, q_h = rk.cpu().numpy(), rv.cpu().numpy(), q.cpu().numpy()
    out_h, plain_h = out.float().cpu().numpy(), out_plain.float().cpu().numpy()
    starts = _starts(w.lens)
    for s, L in enumerate(w.lens):
        k_hat, v_hat = [], []
        for h in range(2):
            rows_k = rk_h[starts[s]:starts[s] + L, h]
            rows_v = rv_h[starts[s]:starts[s] + L, h]
            tk, tail_k = o.quantize_sequence(rows_k, w.tile_tokens, w.bits_k, w.iters, dtype=np.float32, seed=SEED)
            tv, tail_v = o.quantize_sequence(rows_v, w.tile_tokens, w.bits_v, w.iters, dtype=np.float32, seed=SEED)
            k_hat.append(o.sequence_kv_hat(tk, tail_k, SEED))
            v_hat.append(o.sequence_kv_hat(tv, tail_v, SEED))
        ref = o.decode_sequence(q_h[s].astype(np.float64), k_hat, v_hat, w.group_size)
        for hq in range(w.num_q_heads):
            assert rel_l2(out_h[s, hq], ref[hq]) <= ATTN_REL_L2_MAX, (s, hq)
        if L >= w.tile_tokens:  # sequences with quantized tiles
            assert rel_l2(plain_h[s], ref) > 1e-2


def test_seeded_append_equals_prefill():
    t = 64
    chunks = [1] * 40 + [100, 3]
    l0 = 2 * t + 5
    total = l0 + sum(chunks)
    w = synth.workload("qwen3_32b_burst", num_seqs=2, lens=(l0, l0), num_kv_heads=2, group_size=4, tile_tokens=t)
    cfg, a = _cache(w, SEED, extra_tokens=total)
    _, b = _cache(w, SEED, extra_tokens=total)
    rk = synth.kv_rows(w, "k", 2 * total, device="cuda")
    rv = synth.kv_rows(w, "v", 2 * total, device="cuda")
    a.prefill(rk[:2 * l0], rv[:2 * l0], [l0, l0])
    pos = 2 * l0
    for c in chunks:
        a.append(rk[pos:pos + 2 * c], rv[pos:pos + 2 * c], counts=[c, c])
        pos += 2 * c
    # the same tokens per sequence in order, prefilled at once
    idx = [np.arange(s * l0, (s + 1) * l0) for s in range(2)]
    p = 2 * l0
    for c in chunks:
        for s in range(2):
            idx[s] = np.concatenate([idx[s], np.arange(p + s * c, p + (s + 1) * c)])
        p += 2 * c
    order = torch.from_numpy(np.concatenate(idx)).cuda()
    b.prefill(rk.index_select(0, order), rv.index_select(0, order), [total, total])
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool)
    n_tail = total % t
    assert torch.equal(a.k_tail[:, :, :n_tail], b.k_tail[:, :, :n_tail])
