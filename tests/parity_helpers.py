"""Helpers shared by the GPU parity tests: oracle pipelines over the same
seeded inputs the CUDA path gets, and the comparison metrics.

Tolerances (stated once, used by every parity test):
  codes         >= 99.99 % identical, the rest off by exactly 1, and every
                differing code a rounding tie: the fp64 value
                v = (Y_ij - z_i) / s_i lies within
                delta_ij = TIE_EPS (|Y_ij| + |z_i|) / s_i of a half-integer
                and both codes are floor(v) or floor(v) + 1 (both sides take
                the code decision in float32, in different orders)
  s~, z~, C~    within 1 fp16 ulp, and every differing value a rounding tie:
                the fp64 value (s R, z R or C) lies within TIE_EPS * amp * |x|
                of the midpoint of the two fp16 values (amp =
                (|max_j Y| + |z|) / (max_j Y - z) for s~, 1 for z~ and C~)
  dequantized   |X^'_gpu - X^'_oracle| <= s~_i C~_j (one quantization step)
                plus the fp16 rounding of the metadata
  attention     relative L2 error <= 1e-3 per (sequence, query head)
  tails         bit-exact
"""

from __future__ import annotations

import math

import numpy as np
import torch

from oracle import kvq_oracle as o
from quantized_paged_kv_tile_b200 import kvq, synth

CODE_MATCH_MIN = 0.9999
ATTN_REL_L2_MAX = 1e-3
# Relative float32 error allowed at a rounding tie: 2^-17 = 128 u (u = 2^-24).
# The float32 oracle itself stays within 7.3 u (codes, relative to
# (|Y| + |z|) / s) and 11 u (s R, z R, C) of fp64 on the workloads' inputs at
# n = 1..8; a second float32 implementation in another summation order has an
# error of the same kind, so a decision the two sides take differently must
# sit within the sum of both errors of the rounding boundary.
TIE_EPS = 2.0 ** -17


def fp16_ulp_distance(a, b) -> np.ndarray:
    """|a - b| in units of fp16 ulps (ordered-integer distance of the bit patterns)."""
    def ordered(x):
        u = np.asarray(x, dtype=np.float16).view(np.int16).astype(np.int32)
        return np.where(u < 0, -32768 - u, u)
    return np.abs(ordered(a) - ordered(b))


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def make_cache(w: synth.Workload, extra_tokens: int = 0, device="cuda", num_splits: int = 0):
    from quantized_paged_kv_tile_b200.paged import PagedKVCache
    cfg = kvq.Config(num_kv_heads=w.num_kv_heads, group_size=w.group_size, tile_tokens=w.tile_tokens,
                     bits_k=w.bits_k, bits_v=w.bits_v, iters=w.iters, head_dim=w.head_dim)
    max_tokens = max(w.lens) + max(extra_tokens, w.append_tokens)
    bps = -(-max(max_tokens, 1) // 16)
    cache = PagedKVCache(cfg, w.num_seqs, bps * 16, device=device, block_table=synth.block_table(w, bps),
                         num_splits=num_splits)
    return cfg, cache


def unpack_all(cfg: kvq.Config, cache, tiles, is_v: bool):
    """GPU read-back of (seq, tile) pairs: codes, meta, cvec, out_rot as numpy."""
    n, h, t, d = len(tiles), cfg.num_kv_heads, cfg.tile_tokens, cfg.head_dim
    dev = cache.device
    desc = torch.tensor(np.asarray(tiles, dtype=np.int32).reshape(-1, 2), device=dev)
    codes = torch.empty((n, h, t, d), dtype=torch.uint8, device=dev)
    meta = torch.empty((n, h, t, 2), dtype=torch.float16, device=dev)
    cvec = torch.empty((n, h, d), dtype=torch.float16, device=dev)
    rot = torch.empty((n, h, t, d), dtype=torch.float32, device=dev)
    orig = torch.empty((n, h, t, d), dtype=torch.float32, device=dev)
    pool = cache.v_pool if is_v else cache.k_pool
    kvq.unpack_tiles(cfg, desc, cache.block_tables, pool, is_v, codes=codes, meta=meta, cvec=cvec, out_rot=rot,
                     out_orig=orig, num_blocks=cache.num_blocks, dev_status=cache.dev_status)
    return {k: v.cpu().numpy() for k, v in
            dict(codes=codes, meta=meta, cvec=cvec, rot=rot, orig=orig).items()}


class TileStats:
    """Accumulates the quantize comparison of GPU tiles with the float32
    oracle.  ``add`` takes ``src = (rows, bits, iters, seed)``, the raw fp16
    tile the GPU quantized: every code or metadata value that differs from the
    oracle is then checked to be a rounding tie against the fp64 oracle."""

    def __init__(self):
        self.codes = 0
        self.equal = 0
        self.max_code_diff = 0
        self.max_meta_ulp = 0
        self.max_c_ulp = 0
        self.deq_violations = 0
        self.tiles = 0
        self.exact_tiles = 0
        self.code_diffs = 0       # differing codes, all checked for ties
        self.meta_diffs = 0       # differing s~, z~, C~ values, all checked for ties
        self.untied = []          # differences that are not rounding ties
        self.unchecked = 0        # tiles with differences and no source rows

    def add(self, gpu_codes, gpu_meta, gpu_c, gpu_rot, ref: dict, src=None):
        diff = np.abs(gpu_codes.astype(np.int32) - ref["codes"].astype(np.int32))
        self.codes += diff.size
        self.equal += int((diff == 0).sum())
        self.max_code_diff = max(self.max_code_diff, int(diff.max()))
        mu = max(int(fp16_ulp_distance(gpu_meta[:, 0], ref["s_t"]).max()),
                 int(fp16_ulp_distance(gpu_meta[:, 1], ref["z_t"]).max()))
        self.max_meta_ulp = max(self.max_meta_ulp, mu)
        cu = int(fp16_ulp_distance(gpu_c, ref["c_t"]).max())
        self.max_c_ulp = max(self.max_c_ulp, cu)
        ref_rot, _ = o.dequantize_tile(ref["codes"], ref["s_t"], ref["z_t"], ref["c_t"])
        s = np.maximum(np.abs(gpu_meta[:, 0].astype(np.float64)), np.abs(ref["s_t"].astype(np.float64)))
        z = np.maximum(np.abs(gpu_meta[:, 1].astype(np.float64)), np.abs(ref["z_t"].astype(np.float64)))
        c = np.maximum(np.abs(gpu_c.astype(np.float64)), np.abs(ref["c_t"].astype(np.float64)))
        qmax = float(ref["codes"].max()) if ref["codes"].size else 0.0
        step = s[:, None] * c[None, :]
        meta_slack = 2.0 ** -10 * (s[:, None] * max(qmax, 1.0) + z[:, None]) * c[None, :] * 2
        bound = step * (1 + 2.0 ** -9) + meta_slack + 1e-30
        self.deq_violations += int((np.abs(gpu_rot - ref_rot) > bound).sum())
        self.tiles += 1
        if diff.max() == 0 and mu == 0 and cu == 0:
            self.exact_tiles += 1
            return
        if src is None:
            self.unchecked += 1
            return
        self._check_ties(gpu_codes, gpu_meta, gpu_c, ref, diff, src)

    def _check_ties(self, gpu_codes, gpu_meta, gpu_c, ref, diff, src):
        rows, bits, iters, seed = src
        p = o.quantize_tile(rows, bits, iters, dtype=np.float64, return_parts=True, seed=seed)
        y, s, z = p["y"], p["s"], p["z"]
        qmax = (1 << bits) - 1
        ii, jj = np.nonzero(diff)
        self.code_diffs += ii.size
        for i, j in zip(ii, jj):
            if not s[i] > 0:
                self.untied.append(("code on a constant row", i, j))
                continue
            v = (y[i, j] - z[i]) / s[i]
            lo = math.floor(v)
            delta = TIE_EPS * (abs(y[i, j]) + abs(z[i])) / s[i]
            pair = {min(max(lo, 0), qmax), min(max(lo + 1, 0), qmax)}
            if abs(v - lo - 0.5) > delta or int(gpu_codes[i, j]) not in pair or int(ref["codes"][i, j]) not in pair:
                self.untied.append(("code", i, j, v, delta, int(gpu_codes[i, j]), int(ref["codes"][i, j])))
        ymax = y.max(axis=1)
        amp_s = (np.abs(ymax) + np.abs(z)) / np.where(ymax > z, ymax - z, 1.0)
        for name, gpu_v, ref_v, exact, amp in (("s~", gpu_meta[:, 0], ref["s_t"], s * p["r"], amp_s),
                                               ("z~", gpu_meta[:, 1], ref["z_t"], z * p["r"], None),
                                               ("C~", gpu_c, ref["c_t"], p["c"], None)):
            differ = np.nonzero(np.asarray(gpu_v).view(np.uint16) != np.asarray(ref_v).view(np.uint16))[0]
            self.meta_diffs += differ.size
            for k in differ:
                a, b = float(gpu_v[k]), float(ref_v[k])
                mid = 0.5 * (a + b)
                tol = TIE_EPS * (1.0 if amp is None else float(amp[k])) * abs(float(exact[k]))
                if abs(float(exact[k]) - mid) > tol:
                    self.untied.append((name, int(k), float(exact[k]), a, b))

    def check(self):
        frac = self.equal / max(self.codes, 1)
        assert frac >= CODE_MATCH_MIN, f"code match {frac:.6f} < {CODE_MATCH_MIN}"
        assert self.max_code_diff <= 1, f"max code diff {self.max_code_diff}"
        assert self.max_meta_ulp <= 1, f"meta differs by {self.max_meta_ulp} fp16 ulps"
        assert self.max_c_ulp <= 1, f"C differs by {self.max_c_ulp} fp16 ulps"
        assert self.deq_violations == 0, f"{self.deq_violations} dequantized values off by more than one step"
        assert self.unchecked == 0, f"{self.unchecked} tiles differ from the oracle without a tie check"
        assert not self.untied, f"{len(self.untied)} differences are not rounding ties: {self.untied[:5]}"
        return frac


def oracle_tile(rows: np.ndarray, bits: int, iters: int, seed: int = 0) -> dict:
    """Oracle quantization of one T x d tile, taking the code decision in float32."""
    return o.quantize_tile(rows, bits, iters, dtype=np.float32, seed=seed)


def compare_sequence_tiles(cfg: kvq.Config, cache, rows_k: np.ndarray, rows_v: np.ndarray, starts, tiles,
                           stats_k: TileStats, stats_v: TileStats):
    """Check every (seq, tile) of ``tiles`` for every KV head against the oracle.
    rows_* are the packed fp16 rows [N][H_kv][d] on the host."""
    t = cfg.tile_tokens
    gk = unpack_all(cfg, cache, tiles, False)
    gv = unpack_all(cfg, cache, tiles, True)
    for n, (s, ti) in enumerate(tiles):
        r0 = starts[s] + ti * t
        for h in range(cfg.num_kv_heads):
            for rows, g, bits, st in ((rows_k, gk, cfg.bits_k, stats_k), (rows_v, gv, cfg.bits_v, stats_v)):
                tile = rows[r0:r0 + t, h]
                ref = oracle_tile(tile, bits, cfg.iters, cfg.rotation_seed)
                st.add(g["codes"][n, h], g["meta"][n, h], g["cvec"][n, h], g["rot"][n, h], ref,
                       src=(tile, bits, cfg.iters, cfg.rotation_seed))


def oracle_decode_sequence(cfg: kvq.Config, rows_k: np.ndarray, rows_v: np.ndarray, q: np.ndarray,
                           scale: float | None = None) -> np.ndarray:
    """fp64 decode of one sequence from its raw rows [L][H_kv][d] (quantized
    by the oracle tile by tile, tail raw) for queries q [H_q][d]."""
    k_hat, v_hat = [], []
    for h in range(cfg.num_kv_heads):
        tk, tail_k = o.quantize_sequence(rows_k[:, h], cfg.tile_tokens, cfg.bits_k, cfg.iters, dtype=np.float32)
        tv, tail_v = o.quantize_sequence(rows_v[:, h], cfg.tile_tokens, cfg.bits_v, cfg.iters, dtype=np.float32)
        k_hat.append(o.sequence_kv_hat(tk, tail_k))
        v_hat.append(o.sequence_kv_hat(tv, tail_v))
    return o.decode_sequence(q.astype(np.float64), k_hat, v_hat, cfg.group_size, scale)


def gpu_pages_kv_hat(cfg: kvq.Config, cache, seq: int, head: int, length: int, is_v: bool) -> np.ndarray:
    """Original-domain K^ (or V^) of (seq, head) over the first ``length``
    tokens as the GPU stored them: its pages read back by the oracle's own
    page reader, then the raw tail."""
    t, p = cfg.tile_tokens, cfg.page_tokens
    n_full, tau = length // t, length % t
    bits = cfg.bits_v if is_v else cfg.bits_k
    pool = cache.v_pool if is_v else cache.k_pool
    ids = cache.block_tables[seq, :n_full * (t // p)].long()
    host = pool.index_select(0, ids)[:, head:head + 1].cpu().numpy()
    tiles = [o.read_tile_pages(host, range(i * (t // p), (i + 1) * (t // p)), 0, bits, t, is_v, d=cfg.head_dim)
             for i in range(n_full)]
    tail = (cache.v_tail if is_v else cache.k_tail)[seq, head, :tau].cpu().numpy()
    return o.sequence_kv_hat(tiles, tail, cfg.rotation_seed)


def decode_over_gpu_pages(cfg: kvq.Config, cache, seq: int, length: int, q_heads: np.ndarray) -> np.ndarray:
    """fp64 attention of every query head of ``seq`` over the GPU's own pages
    (isolates the read path from the write path)."""
    k_hat = [gpu_pages_kv_hat(cfg, cache, seq, h, length, False) for h in range(cfg.num_kv_heads)]
    v_hat = [gpu_pages_kv_hat(cfg, cache, seq, h, length, True) for h in range(cfg.num_kv_heads)]
    return o.decode_sequence(np.asarray(q_heads, dtype=np.float64), k_hat, v_hat, cfg.group_size)
