"""A serving step (append one token per sequence, then decode) captured in a
CUDA graph and replayed gives, step by step, exactly the eager calls'
outputs, pages and tails, across tile completions inside the graph."""

import numpy as np
import pytest
import torch

from quantized_paged_kv_tile_b200 import kvq, synth
from quantized_paged_kv_tile_b200.paged import DecodeStepGraph

from parity_helpers import make_cache

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("t,splits,fused", [(64, 0, False), (128, 3, False), (64, 5, True), (128, 2, True)])
def test_graph_step_equals_eager(t, splits, fused):
    kvq.load_library()
    steps = 70
    w = synth.workload("qwen3_32b_burst", num_seqs=2, lens=(2 * t + 2, t - 3), num_kv_heads=2, group_size=4,
                       tile_tokens=t)
    _, a = make_cache(w, extra_tokens=steps, num_splits=splits)
    _, b = make_cache(w, extra_tokens=steps, num_splits=splits)
    total = int(sum(w.lens))
    rk = synth.kv_rows(w, "k", total, device="cuda")
    rv = synth.kv_rows(w, "v", total, device="cuda")
    a.prefill(rk, rv, w.lens)
    b.prefill(rk, rv, w.lens)
    graph = DecodeStepGraph(b, num_splits=splits if fused else None, fused=fused)
    fused_steps = 0
    for i in range(steps):
        nk = synth.kv_rows(w, "k", w.num_seqs, device="cuda", stream_id=1 + i)
        nv = synth.kv_rows(w, "v", w.num_seqs, device="cuda", stream_id=1 + i)
        q = synth.queries(w, device="cuda", step=i)
        a.append(nk, nv)
        out_a = a.decode(q)
        graph.new_k.copy_(nk)
        graph.new_v.copy_(nv)
        graph.q.copy_(q)
        fused_steps += fused and not graph.completes_tile()
        out_b = graph.replay()
        assert torch.equal(out_a, out_b), i
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    assert torch.equal(a.seq_lens, b.seq_lens)
    np.testing.assert_array_equal(a.host_lens, b.host_lens)
    assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool)
    assert torch.equal(a.k_tail, b.k_tail) and torch.equal(a.v_tail, b.v_tail)
    if fused:  # every step that completes no tile went through the one-launch step, whose workspace stays zero
        completing = sum(any((n + i + 1) % t == 0 for n in w.lens) for i in range(steps))
        assert 0 < completing < steps and fused_steps == steps - completing
        # the counters (unit queue, CTA count, per-(sequence, KV head) arrivals)
        # are back at zero; the records after them hold the last step's partials
        ws = graph.step_workspace.view(torch.int32)
        B, H = w.num_seqs, w.num_kv_heads
        arrivals = (16 + 4 * (B + 1) + 4 * B) // 4
        assert not ws[:3].any() and not ws[arrivals:arrivals + B * H].any()


def test_fused_step_two_level_merge():
    # 40 chunks per (sequence, KV head): the one-launch step merges groups of
    # 16 chunks, then the groups, and equals append + decode with the same
    # split count bit for bit, step after step
    kvq.load_library()
    w = synth.workload("tiny", num_seqs=2, lens=(64 * 40 + 3, 64 * 17 + 9), num_kv_heads=2, group_size=4)
    cfg, a = make_cache(w, extra_tokens=8, num_splits=40)
    _, b = make_cache(w, extra_tokens=8, num_splits=40)
    total = int(sum(w.lens))
    rk = synth.kv_rows(w, "k", total, device="cuda")
    rv = synth.kv_rows(w, "v", total, device="cuda")
    a.prefill(rk, rv, w.lens)
    b.prefill(rk, rv, w.lens)
    ws = torch.zeros(kvq.decode_workspace_bytes(cfg, 2, 40), dtype=torch.uint8, device="cuda")
    for i in range(8):
        nk = synth.kv_rows(w, "k", 2, device="cuda", stream_id=1 + i)
        nv = synth.kv_rows(w, "v", 2, device="cuda", stream_id=1 + i)
        q = synth.queries(w, device="cuda", step=i)
        a.append(nk, nv)
        out_a = a.decode(q, num_splits=40)
        out_b = torch.empty_like(q)
        kvq.append_decode_step(cfg, nk, nv, q, out_b, b.seq_lens, b.block_tables, b.k_pool, b.v_pool, b.k_tail,
                               b.v_tail, ws, 40, num_blocks=b.num_blocks, dev_status=b.dev_status)
        assert torch.equal(out_a, out_b), i
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    assert torch.equal(a.seq_lens, b.seq_lens)
    assert torch.equal(a.k_tail, b.k_tail) and torch.equal(a.v_tail, b.v_tail)


def test_fused_step_refuses_a_tile_completion():
    # a token that completes a tile must be quantized into pages, which the
    # one-launch step does not do: it is reported and not written
    kvq.load_library()
    w = synth.workload("tiny", num_seqs=2, lens=(63, 40), num_kv_heads=1, group_size=2)
    cfg, c = make_cache(w, extra_tokens=2)
    rk = synth.kv_rows(w, "k", 103, device="cuda")
    rv = synth.kv_rows(w, "v", 103, device="cuda")
    c.prefill(rk, rv, [63, 40])
    ws = torch.zeros(kvq.decode_workspace_bytes(cfg, 2, 2), dtype=torch.uint8, device="cuda")
    nk = torch.ones((2, 1, 128), dtype=torch.float16, device="cuda")
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


def test_graph_refuses_step_past_the_pages():
    kvq.load_library()
    w = synth.workload("tiny", num_seqs=1, lens=(30,), num_kv_heads=1, group_size=2)
    _, c = make_cache(w, extra_tokens=2)  # room for exactly 2 more tokens
    rk = synth.kv_rows(w, "k", 30, device="cuda")
    rv = synth.kv_rows(w, "v", 30, device="cuda")
    c.prefill(rk, rv, [30])
    graph = DecodeStepGraph(c)
    graph.replay()
    graph.replay()
    with pytest.raises(ValueError):
        graph.replay()
