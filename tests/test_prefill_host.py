"""CPU checks of the chunked-prefill host path: argument validation in
PagedKVCache.prefill_chunk and the binding, and that nothing falls back to
the CPU (a call with CPU tensors is refused before the library)."""

import numpy as np
import pytest
import torch

from quantized_paged_kv_tile_b200 import build, kvq
from quantized_paged_kv_tile_b200.paged import PagedKVCache


@pytest.fixture(scope="module")
def cache():
    build.build()
    cfg = kvq.Config(num_kv_heads=2, group_size=4, tile_tokens=64, bits_k=4, bits_v=4, iters=2)
    # an explicit split count keeps the constructor off the device query
    return PagedKVCache(cfg, 2, 256, device="cpu", num_splits=2)


def _rows(n, heads):
    return torch.zeros((n, heads, 128), dtype=torch.float16)


def test_counts_must_match_sequences(cache):
    q, k = _rows(3, 8), _rows(3, 2)
    with pytest.raises(ValueError):
        cache.prefill_chunk(q, k, k, [3])              # one count for two sequences
    with pytest.raises(ValueError):
        cache.prefill_chunk(q, k, k, [4, -1])          # negative count


def test_append_past_pages_is_refused(cache):
    q, k = _rows(300, 8), _rows(300, 2)
    with pytest.raises(ValueError):
        cache.prefill_chunk(q, k, k, [0, 300])         # 256 tokens per sequence allocated
    assert list(cache.host_lens) == [0, 0]


def test_no_cpu_fallback(cache):
    q, k = _rows(2, 8), _rows(2, 2)
    with pytest.raises(TypeError, match="CUDA tensor"):
        cache.prefill_chunk(q, k, k, [1, 1], append=False)
    assert list(cache.host_lens) == [0, 0]
