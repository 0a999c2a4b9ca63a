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


@pytest.mark.parametrize("t,splits", [(64, 0), (128, 3)])
def test_graph_step_equals_eager(t, splits):
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
    graph = DecodeStepGraph(b)
    for i in range(steps):
        nk = synth.kv_rows(w, "k", w.num_seqs, device="cuda", stream_id=1 + i)
        nv = synth.kv_rows(w, "v", w.num_seqs, device="cuda", stream_id=1 + i)
        q = synth.queries(w, device="cuda", step=i)
        a.append(nk, nv)
        out_a = a.decode(q)
        graph.new_k.copy_(nk)
        graph.new_v.copy_(nv)
        graph.q.copy_(q)
        out_b = graph.replay()
        assert torch.equal(out_a, out_b), i
    torch.cuda.synchronize()
    assert a.status() == 0 and b.status() == 0
    assert torch.equal(a.seq_lens, b.seq_lens)
    np.testing.assert_array_equal(a.host_lens, b.host_lens)
    assert torch.equal(a.k_pool, b.k_pool) and torch.equal(a.v_pool, b.v_pool)
    assert torch.equal(a.k_tail, b.k_tail) and torch.equal(a.v_tail, b.v_tail)


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
