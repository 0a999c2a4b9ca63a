"""Seeded synthetic workloads (shapes, value distributions, page scatter).

This module holds no arithmetic of the method: it only draws random
numbers with the shapes and distributions of the five workloads below.
Both the CUDA path and the CPU oracle take their inputs from here.

Workloads (sizes and distributions as specified for this project):
  tiny            1 seq x 1024 tokens, 1 KV head, 8 query heads, T=64, b=4/4,
                  n=4; K, V ~ N(0,1) with 4 seeded channels x20 (same 4 for
                  K and V); one decode query ~ N(0,1).
  qwen3_4b        Qwen3-4B-shaped layer: 6 seqs x 131072 tokens (+1 appended),
                  8 KV heads, 32 query heads, T=64, b=4/4, n=4.  K channel
                  std ~ lognormal(0,1) per (head, channel) plus 2% outlier
                  channels x10; V ~ N(0,1).  Stand-in for the 128K-context
                  Qwen3-4B runs on aitrends.kr article 74976 ("TL;DR").
  qwen3_32b_burst Qwen3-32B-shaped burst: 64 seqs x 16384 tokens, 8 KV heads,
                  64 query heads, T=128, b=4 K / 2 V, n=2, 1024 decode steps
                  appending one token each; distributions as qwen3_4b.
                  Stand-in for the 16K-context burst on the axbrief.com
                  KVarN article (lead section).
  prefill_sweep   32 seqs x 16384 new tokens, 8 KV heads; per head 1-5% of
                  channels scaled by log-uniform [5, 50], for K and V;
                  T in {32,64,128} x b in {2,3,4} x n in {1,4,8}.
  mixed           256 seqs, lengths floor(exp(U(ln 1024, ln 131072))), 8 KV
                  heads, 64 query heads, T=64, b=4 K / 2 V, n=4.
Seeds: workload k uses numpy PCG64(1000 + k) for the small per-channel
draws and torch generators seeded from it for the bulk N(0,1) draws; the
page scatter (block-table permutation) uses PCG64(2000 + k).
"""

from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

HEAD_DIM = 128
PAGE_TOKENS = 16


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int                 # 1-based workload number (seed 1000 + index)
    num_seqs: int
    num_kv_heads: int
    group_size: int
    tile_tokens: int
    bits_k: int
    bits_v: int
    iters: int
    kv_dist: str               # "tiny" | "lognormal" | "sweep"
    lens: tuple = ()           # cached tokens per sequence (before appends)
    append_tokens: int = 0     # tokens appended per sequence by the step
    decode_steps: int = 1
    replica: int = 0           # independent replica batch (multi-GPU weak scaling)
    head_dim: int = HEAD_DIM   # d: 128 in every named workload; 64 and 256 for the variant tests

    @property
    def seed(self) -> int:
        return 1000 + self.index + 7919 * self.replica

    @property
    def table_seed(self) -> int:
        return 2000 + self.index + 7919 * self.replica

    @property
    def num_q_heads(self) -> int:
        return self.num_kv_heads * self.group_size


def mixed_lengths(num_seqs: int = 256, seed: int = 1005, lo: int = 1024, hi: int = 131072) -> tuple:
    rng = np.random.Generator(np.random.PCG64(seed))
    u = rng.uniform(math.log(lo), math.log(hi), size=num_seqs)
    return tuple(int(x) for x in np.floor(np.exp(u)))


def workload(name: str, **overrides) -> Workload:
    """The named workload; keyword overrides give smaller test variants."""
    base = {
        "tiny": dict(index=1, num_seqs=1, num_kv_heads=1, group_size=8, tile_tokens=64, bits_k=4, bits_v=4,
                     iters=4, kv_dist="tiny", lens=(1024,), append_tokens=0),
        "qwen3_4b": dict(index=2, num_seqs=6, num_kv_heads=8, group_size=4, tile_tokens=64, bits_k=4, bits_v=4,
                         iters=4, kv_dist="lognormal", lens=(131072,) * 6, append_tokens=1),
        "qwen3_32b_burst": dict(index=3, num_seqs=64, num_kv_heads=8, group_size=8, tile_tokens=128, bits_k=4,
                                bits_v=2, iters=2, kv_dist="lognormal", lens=(16384,) * 64, append_tokens=1,
                                decode_steps=1024),
        "prefill_sweep": dict(index=4, num_seqs=32, num_kv_heads=8, group_size=8, tile_tokens=64, bits_k=4,
                              bits_v=4, iters=4, kv_dist="sweep", lens=(16384,) * 32, append_tokens=0),
        "mixed": dict(index=5, num_seqs=256, num_kv_heads=8, group_size=8, tile_tokens=64, bits_k=4, bits_v=2,
                      iters=4, kv_dist="lognormal", lens=mixed_lengths(), append_tokens=1),
    }[name]
    base.update(overrides)
    if "lens" in overrides or "num_seqs" in overrides:
        lens = tuple(base["lens"])
        if len(lens) != base["num_seqs"]:
            lens = (lens + lens * base["num_seqs"])[: base["num_seqs"]]
        base["lens"] = lens
    return Workload(name=name, **base)


def channel_scales(w: Workload, which: str) -> np.ndarray:
    """Per (KV head, channel) multipliers of the N(0,1) draws, float32 [H_kv][d]."""
    salt = {"k": 11, "v": 23}[which]
    rng = np.random.Generator(np.random.PCG64([w.seed, salt]))
    h, d = w.num_kv_heads, w.head_dim
    if w.kv_dist == "tiny":
        # the same 4 channels for K and V: draw them from a stream shared by both
        shared = np.random.Generator(np.random.PCG64([w.seed, 5]))
        ch = shared.choice(d, size=4, replace=False)
        sc = np.ones((h, d), dtype=np.float32)
        sc[:, ch] = 20.0
        return sc
    if w.kv_dist == "lognormal":
        if which == "v":
            return np.ones((h, d), dtype=np.float32)
        sc = rng.lognormal(0.0, 1.0, size=(h, d)).astype(np.float32)
        n_out = math.ceil(0.02 * d)
        for head in range(h):
            sc[head, rng.choice(d, size=n_out, replace=False)] *= 10.0
        return sc
    if w.kv_dist == "sweep":
        sc = np.ones((h, d), dtype=np.float32)
        for head in range(h):
            f = rng.uniform(0.01, 0.05)
            k = max(1, int(round(f * d)))
            ch = rng.choice(d, size=k, replace=False)
            sc[head, ch] = np.exp(rng.uniform(math.log(5.0), math.log(50.0), size=k))
        return sc
    raise ValueError(w.kv_dist)


def _generator(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def kv_rows(w: Workload, which: str, num_rows: int, device="cpu", stream_id: int = 0) -> torch.Tensor:
    """fp16 [num_rows][H_kv][d]: N(0,1) times the channel multipliers.

    ``stream_id`` selects an independent stream (0 = the cached prefix,
    1.. = appended tokens of later steps)."""
    salt = {"k": 1, "v": 2}[which]
    g = _generator(device, (w.seed * 1000 + salt) * 4099 + stream_id)
    x = torch.randn((num_rows, w.num_kv_heads, w.head_dim), generator=g, device=device, dtype=torch.float32)
    x *= torch.from_numpy(channel_scales(w, which)).to(device)[None]
    return x.to(torch.float16)


def kv_rows_one_head(w: Workload, which: str, num_rows: int, head: int, stream_id: int = 0) -> np.ndarray:
    """fp16 [num_rows][d] for one KV head, on the host, from its own seeded
    stream (same distribution as ``kv_rows``; used by CPU baselines that
    need one head of a long sequence without drawing all heads)."""
    salt = {"k": 1, "v": 2}[which]
    rng = np.random.Generator(np.random.PCG64([w.seed, salt, head, stream_id]))
    x = rng.standard_normal((num_rows, w.head_dim), dtype=np.float32)
    x *= channel_scales(w, which)[head][None, :]
    return x.astype(np.float16)


def queries(w: Workload, device="cpu", step: int = 0) -> torch.Tensor:
    """fp16 [B][H_q][d] ~ N(0,1)."""
    g = _generator(device, (w.seed * 1000 + 3) * 4099 + step)
    return torch.randn((w.num_seqs, w.num_q_heads, w.head_dim), generator=g, device=device,
                       dtype=torch.float32).to(torch.float16)


def block_table(w: Workload, blocks_per_seq: int, extra_blocks: int = 0) -> np.ndarray:
    """int32 [B][blocks_per_seq]: a seeded permutation of all physical blocks,
    so logically adjacent pages are scattered over the pool."""
    rng = np.random.Generator(np.random.PCG64(w.table_seed))
    total = w.num_seqs * blocks_per_seq + extra_blocks
    perm = rng.permutation(total)[: w.num_seqs * blocks_per_seq]
    return perm.reshape(w.num_seqs, blocks_per_seq).astype(np.int32)
