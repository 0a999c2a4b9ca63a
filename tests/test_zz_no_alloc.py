"""Decode on the library's static scratch (kvq_paged_decode_attention_static_scratch).

The entry point allocates nothing: its workspace is a device array built into
the library, one per device, looked up on the first call.  This file sorts
last so that its GPU test runs both after the rest of the suite and, when
selected alone, in a fresh process where its first call does the look-up.
"""

import ctypes

import numpy as np
import pytest
import torch

from parity_helpers import make_cache
from quantized_paged_kv_tile_b200 import build, kvq, synth


def test_static_scratch_size_matches_header():
    text = open(kvq.__file__.replace("quantized_paged_kv_tile_b200/kvq.py", "include/kvq.h")).read()
    assert "#define KVQ_DECODE_STATIC_SCRATCH_BYTES ((size_t)32 << 20)" in text
    assert kvq.DECODE_STATIC_SCRATCH_BYTES == 32 << 20


def test_static_scratch_rejects_oversize_before_the_device():
    # an explicit split count keeps the size computation on the host; the
    # call must fail on the size alone, before any pointer or device access
    build.build()
    lib = kvq.load_library()
    cfg = kvq.Config(num_kv_heads=8, group_size=8, tile_tokens=64, bits_k=4, bits_v=4, iters=4)
    num_seqs, splits = 64, 64
    need = kvq.decode_workspace_bytes(cfg, num_seqs, splits)
    assert need > kvq.DECODE_STATIC_SCRATCH_BYTES
    st = lib.kvq_paged_decode_attention_static_scratch(
        ctypes.byref(cfg.c()), None, None, None, num_seqs, None, 1, 1, None, None, None, None,
        ctypes.c_float(0.088), splits, None, None)
    assert st == kvq.KVQ_ERR_WORKSPACE
    msg = lib.kvq_last_error().decode()
    assert str(need) in msg and str(kvq.DECODE_STATIC_SCRATCH_BYTES) in msg
    # bad arguments are still rejected first
    st = lib.kvq_paged_decode_attention_static_scratch(
        ctypes.byref(cfg.c()), None, None, None, -1, None, 1, 1, None, None, None, None,
        ctypes.c_float(0.088), splits, None, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG


CASES = [
    # (workload overrides, num_splits)
    (dict(num_seqs=3, lens=(700, 64, 30), num_kv_heads=2, group_size=4, bits_v=2), 0),
    (dict(num_seqs=2, lens=(1000, 257), num_kv_heads=2, group_size=8), 3),
]


@pytest.mark.gpu
@pytest.mark.parametrize("over,splits", CASES)
def test_static_scratch_matches_workspace_entry(over, splits):
    w = synth.workload("tiny", **over)
    cfg, cache = make_cache(w, num_splits=splits)
    total = int(sum(w.lens))
    rk = synth.kv_rows(w, "k", total, device="cuda")
    rv = synth.kv_rows(w, "v", total, device="cuda")
    cache.prefill(rk, rv, w.lens)
    q = synth.queries(w, device="cuda")
    ref = cache.decode(q, num_splits=splits)
    torch.cuda.synchronize()
    assert cache.status() == 0
    ref_h = ref.float().cpu().numpy()
    assert np.all(np.isfinite(ref_h))
    outs = [torch.full_like(q, float("nan")) for _ in range(2)]
    for out in outs:  # two calls in a row on the same scratch
        kvq.paged_decode_attention_static_scratch(cfg, q, out, cache.seq_lens, cache.block_tables, cache.k_pool,
                                                  cache.v_pool, cache.k_tail, cache.v_tail, num_splits=splits,
                                                  num_blocks=cache.num_blocks, dev_status=cache.dev_status)
    torch.cuda.synchronize()
    assert cache.status() == 0
    # the same kernels with the same split count on the same inputs: the
    # outputs are bit-identical to the workspace entry point's, on both calls
    for out in outs:
        assert torch.equal(out, ref)
