"""Device-side failure detection, exercised without a fault: the kernels'
bounded mbarrier waits are run on a barrier that nothing arrives at; each
gives up after its limit, the status word reads KVQ_ERR_DEVICE_TIMEOUT, and
the context is still usable afterwards (a quantize + decode matches the
oracle's tolerance and leaves the status clean)."""

import time

import numpy as np
import pytest
import torch

from quantized_paged_kv_tile_b200 import kvq, synth

from parity_helpers import ATTN_REL_L2_MAX, make_cache, oracle_decode_sequence, rel_l2

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_reports():
    kvq.load_library()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.monotonic()
    kvq.selftest_bounded_wait(status)
    torch.cuda.synchronize()
    elapsed = time.monotonic() - t0
    assert int(status.item()) == kvq.KVQ_ERR_DEVICE_TIMEOUT
    assert 5.5 < elapsed < 40.0  # three waits (quantize, decode, prefill) of the kernels' 2 s limit
    # the context keeps working: a normal prefill + decode + chunked prefill afterwards
    w = synth.workload("tiny", lens=(200,))
    cfg, cache = make_cache(w)
    rk = synth.kv_rows(w, "k", 200, device="cuda")
    rv = synth.kv_rows(w, "v", 200, device="cuda")
    cache.prefill(rk, rv, [200])
    q = synth.queries(w, device="cuda")
    out = cache.decode(q)
    torch.cuda.synchronize()
    assert cache.status() == 0
    ref = oracle_decode_sequence(cfg, rk.cpu().numpy(), rv.cpu().numpy(), q.cpu().numpy()[0])
    out_h = out.float().cpu().numpy()[0]
    for h in range(w.num_q_heads):
        assert rel_l2(out_h[h], ref[h]) <= ATTN_REL_L2_MAX
    # a one-token chunk (raw) over the same cache equals that decode with the token appended first
    ck = synth.kv_rows(w, "k", 1, device="cuda", stream_id=4)
    cv = synth.kv_rows(w, "v", 1, device="cuda", stream_id=4)
    pout = cache.prefill_chunk(q, ck, cv, [1], append=True)
    dout = cache.decode(q)
    torch.cuda.synchronize()
    assert cache.status() == 0
    p_h, d_h = pout.float().cpu().numpy()[0], dout.float().cpu().numpy()[0]
    for h in range(w.num_q_heads):
        assert rel_l2(p_h[h], d_h[h]) <= ATTN_REL_L2_MAX

