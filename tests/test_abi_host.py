"""CPU-only checks of the C ABI library and the host-side helpers.

No compute call reaches the GPU here: the library is loaded, its exported
symbols are compared with include/kvq.h, and only host-side entry points
(layout, workspace sizing with an explicit split count, argument
validation that fails before any launch) are called.
"""

import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from oracle import kvq_oracle as o
from quantized_paged_kv_tile_b200 import build, kvq, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return kvq.load_library()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return sorted(set(re.findall(r"KVQ_API\s+[^;(]*?\b(kvq_\w+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert declared_symbols() == sorted(kvq.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", kvq.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted(set(re.findall(r"\bT (kvq_\w+)", out)))
    assert exported == declared_symbols()
    for name in declared_symbols():
        assert hasattr(lib, name)


def test_version_and_status_strings(lib):
    assert kvq.version().startswith("kvq ") and "sm_100a" in kvq.version()
    assert lib.kvq_status_string(kvq.KVQ_ERR_WORKSPACE).decode() == "workspace too small"


@pytest.mark.parametrize("t", [32, 64, 128])
@pytest.mark.parametrize("bk,bv", [(4, 4), (4, 2), (3, 2), (2, 3), (8, 8)])
def test_layout_matches_oracle(lib, t, bk, bv):
    cfg = kvq.Config(num_kv_heads=8, group_size=4, tile_tokens=t, bits_k=bk, bits_v=bv, iters=4)
    lay = kvq.get_layout(cfg)
    ok_, ov = o.page_layout(bk, t), o.page_layout(bv, t)
    assert lay["page_bytes_k"] == ok_["page_bytes"] and lay["page_bytes_v"] == ov["page_bytes"]
    assert lay["codes_bytes_k"] == ok_["codes"] and lay["cslice_off_k"] == ok_["cslice_off"]
    assert lay["cslice_channels"] == ok_["cslice_channels"] and lay["pages_per_tile"] == t // 16
    assert lay["tail_bytes"] == 8 * t * 128 * 2
    assert lay["block_stride_v"] == 8 * ov["page_bytes"]


@pytest.mark.parametrize("d", [64, 256])
@pytest.mark.parametrize("t", [32, 64, 128])
@pytest.mark.parametrize("bk,bv", [(4, 4), (2, 3), (8, 8)])
def test_layout_matches_oracle_other_head_sizes(lib, d, t, bk, bv):
    cfg = kvq.Config(num_kv_heads=3, group_size=4, tile_tokens=t, bits_k=bk, bits_v=bv, iters=4, head_dim=d)
    lay = kvq.get_layout(cfg)
    ok_, ov = o.page_layout(bk, t, d), o.page_layout(bv, t, d)
    assert lay["page_bytes_k"] == ok_["page_bytes"] and lay["page_bytes_v"] == ov["page_bytes"]
    assert lay["codes_bytes_v"] == ov["codes"] and lay["cslice_off_v"] == ov["cslice_off"]
    assert lay["cslice_channels"] == ok_["cslice_channels"] and lay["tail_bytes"] == 3 * t * d * 2


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 96, kvq.KVQ_ERR_UNSUPPORTED), ("tile_tokens", 48, kvq.KVQ_ERR_UNSUPPORTED),
    ("bits_k", 5, kvq.KVQ_ERR_UNSUPPORTED), ("bits_k", 8, kvq.KVQ_ERR_UNSUPPORTED),  # 8 only with bits_v = 8
    ("group_size", 9, kvq.KVQ_ERR_UNSUPPORTED),
    ("iters", -1, kvq.KVQ_ERR_INVALID_ARG), ("std_eps", 0.0, kvq.KVQ_ERR_INVALID_ARG),
    ("page_tokens", 32, kvq.KVQ_ERR_UNSUPPORTED), ("num_kv_heads", 0, kvq.KVQ_ERR_INVALID_ARG),
])
def test_config_validation(lib, field, value, status):
    base = dict(num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=4, bits_v=4, iters=4)
    cfg = kvq.Config(**base)
    cfg = kvq.Config(**{**cfg.__dict__, field: value})
    with pytest.raises(kvq.KvqError) as ei:
        kvq.get_layout(cfg)
    assert ei.value.status == status


def test_argument_errors_launch_nothing(lib):
    cfg = kvq.Config(num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=4, bits_v=4, iters=4)
    c = cfg.c()
    # both sources NULL
    st = lib.kvq_quantize_tiles(ctypes.byref(c), None, None, 10, 16, 1, 16, 1, 4, 8, 16, 16, None, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG
    # misaligned pointer
    st = lib.kvq_quantize_tiles(ctypes.byref(c), 17, None, 10, 16, 1, 16, 1, 4, 8, 16, 16, None, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG and "aligned" in kvq.load_library().kvq_last_error().decode()
    # head sizes 64 and 256: decode and the serving step (to the workspace
    # check here: one split of 2 sequences x 2 KV heads x 4 query heads x
    # (4 + d) floats; 1 sequence for the step)
    for d in (64, 256):
        cd = kvq.Config(num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=4, bits_v=4, iters=4, head_dim=d)
        assert kvq.decode_workspace_bytes(cd, 2, 1) == 2 * 2 * 1 * 4 * (4 + d) * 4
        st = lib.kvq_paged_decode_attention(ctypes.byref(cd.c()), 16, 16, 16, 2, 16, 4, 8, 16, 16, 16, 16, 0.1, 16,
                                            16, 1, None, None)
        assert st == kvq.KVQ_ERR_WORKSPACE
        st = lib.kvq_append_decode_step(ctypes.byref(cd.c()), 16, 16, 16, 16, 16, 1, 16, 4, 8, 16, 16, 16, 16, 0.1,
                                        16, 1 * 2 * 1 * 4 * (4 + d) * 4 - 1, 1, None, None)
        assert st == kvq.KVQ_ERR_WORKSPACE
        st = lib.kvq_append_decode_step(ctypes.byref(cd.c()), 16, 16, 16, 16, 16, 1, 16, 4, 8, 16, 16, 16, 16, 0.1,
                                        16, 1 << 20, 0, None, None)
        assert st == kvq.KVQ_ERR_INVALID_ARG  # split count 0
    # 3-bit pages are read: the call gets past the configuration checks (here
    # to the workspace check, with no device query for an explicit split count)
    c3 = kvq.Config(num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=3, bits_v=4, iters=4).c()
    st = lib.kvq_paged_decode_attention(ctypes.byref(c3), 16, 16, 16, 1, 16, 4, 8, 16, 16, 16, 16, 0.1, 16,
                                        1, 1, None, None)
    assert st == kvq.KVQ_ERR_WORKSPACE
    # workspace too small (explicit split count: no device query)
    need = kvq.decode_workspace_bytes(cfg, 3, 2)
    # schedule header and counters (256 B), one 528-byte raw-tail record per
    # (sequence, KV head, query head), then one 528-byte partial record per
    # (unit, query head): 3 sequences x 2 KV heads x 2 splits x 4 query heads,
    # then one int32 merge-group counter per unit
    assert need == 256 + 3 * 2 * 4 * 132 * 4 + 3 * 2 * 2 * 4 * 132 * 4 + 3 * 2 * 2 * 4
    st = lib.kvq_paged_decode_attention(ctypes.byref(c), 16, 16, 16, 3, 16, 4, 8, 16, 16, 16, 16, 0.1, 16,
                                        need - 1, 2, None, None)
    assert st == kvq.KVQ_ERR_WORKSPACE
    # a split count whose work units would not fit the device's 32-bit counters is refused on the host
    st = lib.kvq_paged_decode_attention(ctypes.byref(c), 16, 16, 16, 60000, 16, 4, 8, 16, 16, 16, 16, 0.1, 16,
                                        1 << 62, 65535, None, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG and "too large" in kvq.load_library().kvq_last_error().decode()
    # zero-sized work is a no-op
    assert lib.kvq_quantize_tiles(ctypes.byref(c), 16, None, 0, None, 0, None, 0, 0, 0, None, None, None,
                                  None) == kvq.KVQ_OK


def test_prefill_argument_errors_launch_nothing(lib):
    cfg = kvq.Config(num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=4, bits_v=4, iters=4)
    c = cfg.c()
    def call(conf, num_seqs=3, max_chunk=40, q=16, scale=0.1, tables=16, splits=1, ws=None, ws_bytes=0):
        return lib.kvq_paged_prefill_attention(ctypes.byref(conf), q, 16, 16, 16, 16, 16, num_seqs, max_chunk,
                                               tables, 4, 8, 16, 16, 16, 16, scale, splits, ws, ws_bytes, None,
                                               None)
    # head sizes 64 and 256: one launch over the whole context, no workspace
    # for any split count (checked, then ignored); argument errors as at d = 128
    for d in (64, 256):
        cfg_d = kvq.Config(num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=4, bits_v=4, iters=4, head_dim=d)
        assert all(kvq.prefill_workspace_bytes(cfg_d, 3, 40, s) == 0 for s in (1, 3, 64))
        c_d = cfg_d.c()
        assert call(c_d, splits=65) == kvq.KVQ_ERR_INVALID_ARG
        assert call(c_d, q=None) == kvq.KVQ_ERR_INVALID_ARG
        assert call(c_d, num_seqs=70000) == kvq.KVQ_ERR_INVALID_ARG
        assert call(c_d, num_seqs=0) == kvq.KVQ_OK
    # 3-bit pages are read: past the configuration checks, to the workspace check
    c3 = kvq.Config(num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=4, bits_v=3, iters=4).c()
    assert call(c3, splits=2, ws=16, ws_bytes=16) == kvq.KVQ_ERR_WORKSPACE
    assert call(c, num_seqs=-1) == kvq.KVQ_ERR_INVALID_ARG
    assert call(c, max_chunk=-2) == kvq.KVQ_ERR_INVALID_ARG
    assert call(c, q=None) == kvq.KVQ_ERR_INVALID_ARG
    assert call(c, q=24) == kvq.KVQ_ERR_INVALID_ARG            # misaligned
    assert call(c, scale=0.0) == kvq.KVQ_ERR_INVALID_ARG
    assert call(c, splits=0) == kvq.KVQ_ERR_INVALID_ARG
    assert call(c, splits=65) == kvq.KVQ_ERR_INVALID_ARG
    # one 528-byte partial record per (sequence, KV head, 128-row tile, split, row)
    assert kvq.prefill_workspace_bytes(cfg, 3, 40, 1) == 0
    need = kvq.prefill_workspace_bytes(cfg, 3, 40, 3)
    assert need == 3 * 2 * 2 * 3 * 128 * 132 * 4                # 40 tokens x g 4 = 160 rows -> 2 row tiles
    assert call(c, splits=3) == kvq.KVQ_ERR_INVALID_ARG        # workspace NULL
    assert call(c, splits=3, ws=16, ws_bytes=need - 1) == kvq.KVQ_ERR_WORKSPACE
    assert str(need) in lib.kvq_last_error().decode()
    assert call(c, tables=None) == kvq.KVQ_ERR_INVALID_ARG
    assert call(c, num_seqs=70000) == kvq.KVQ_ERR_INVALID_ARG
    assert call(c, num_seqs=0) == kvq.KVQ_OK                   # nothing to do
    assert call(c, max_chunk=0) == kvq.KVQ_OK


def test_binding_rejects_cpu_tensors(lib):
    cfg = kvq.Config(num_kv_heads=1, group_size=1, tile_tokens=64, bits_k=4, bits_v=4, iters=1)
    x = torch.zeros((64, 1, 128), dtype=torch.float16)
    with pytest.raises(TypeError):
        kvq.quantize_tiles(cfg, x, None, torch.zeros((1, 3), dtype=torch.int32), torch.zeros((1, 4), dtype=torch.int32),
                           torch.zeros((4, 1, 1152), dtype=torch.uint8), None)


# ------------------------------------------------------------------ synth

def test_synth_is_seeded_and_shaped():
    w = synth.workload("qwen3_4b", num_seqs=2, lens=(256, 256))
    a = synth.kv_rows(w, "k", 64)
    b = synth.kv_rows(w, "k", 64)
    assert a.shape == (64, 8, 128) and a.dtype == torch.float16
    assert torch.equal(a, b)
    assert not torch.equal(a, synth.kv_rows(w, "v", 64))
    sc = synth.channel_scales(w, "k")
    # 3 outlier channels per head scaled by 10 on top of lognormal(0,1)
    assert sc.shape == (8, 128) and np.all(sc > 0)
    assert np.all(synth.channel_scales(w, "v") == 1.0)


def test_synth_tiny_uses_same_outlier_channels_for_k_and_v():
    w = synth.workload("tiny")
    k, v = synth.channel_scales(w, "k"), synth.channel_scales(w, "v")
    assert (k == 20).sum() == 4 and np.array_equal(k, v)


def test_synth_sweep_outlier_counts():
    w = synth.workload("prefill_sweep")
    for which in ("k", "v"):
        sc = synth.channel_scales(w, which)
        n = (sc != 1.0).sum(axis=1)
        assert np.all(n >= 1) and np.all(n <= 7)
        big = sc[sc != 1.0]
        assert big.min() >= 5.0 and big.max() <= 50.0


def test_mixed_lengths_log_uniform():
    lens = np.array(synth.workload("mixed").lens)
    assert lens.shape == (256,) and lens.min() >= 1024 and lens.max() <= 131072
    # log-uniform: the median sits near the geometric mean of the range
    assert 6000 < np.median(lens) < 24000


def test_block_table_is_a_permutation():
    w = synth.workload("qwen3_4b")
    bt = synth.block_table(w, 8193)
    assert bt.shape == (6, 8193)
    assert np.array_equal(np.sort(bt.ravel()), np.arange(6 * 8193))
    assert not np.array_equal(bt.ravel(), np.arange(6 * 8193))


def test_selftest_rejects_null_status(lib):
    # fails on the host before any launch
    assert lib.kvq_selftest_bounded_wait(None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert "dev_status" in lib.kvq_last_error().decode()


def test_prefill_split_heuristic():
    cfg = kvq.Config(num_kv_heads=8, group_size=4, tile_tokens=64, bits_k=4, bits_v=4, iters=4)
    # one sequence, 512-token chunk: 128 units on 148 SMs -> a split count that fills whole waves
    s = kvq.prefill_splits(cfg, 1, 512, 131073, 148)
    n = 128 * s
    assert n / (-(-n // 148) * 148) >= 0.99 and 2048 // s >= 16
    # six sequences: 768 units (5.19 waves) -> more CTAs
    s6 = kvq.prefill_splits(cfg, 6, 512, 131073, 148)
    n6 = 768 * s6
    assert s6 > 1 and n6 / (-(-n6 // 148) * 148) >= 0.99
    # short contexts are not split (each split keeps >= 16 tiles)
    assert kvq.prefill_splits(cfg, 1, 512, 1500, 148) == 1
    # no chunk tokens: nothing to split
    assert kvq.prefill_splits(cfg, 4, 0, 131073, 148) == 1
