"""Plain CPU oracle for variance-normalized, tile-quantized paged KV caches.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
link this module: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code, constants or helpers with the CUDA library; the only thing
both sides see is the written format specification in ``include/kvq.h``.

What it computes and where the method is stated
-----------------------------------------------
Sources (web pages, cited by title and section):

* [AXB] axbrief.com, "Huawei's KVarN boosts vLLM KV-cache capacity by 5x
  without accuracy loss", section "What differs from existing methods"
  (the four-step paragraph): the cache is quantized in fixed-size token
  tiles; each tile, taken from the raw fp16 cache, gets a Hadamard rotation
  along the channel axis, then Sinkhorn-like iterative variance
  normalization that equalizes the channels' variances, then asymmetric
  round-to-nearest to a low bit width.
* [AIT] aitrends.kr article 74976, "TL;DR" and the glossary entries
  "KV compression" / "attention backend": attention reads the compressed
  pages directly instead of re-materialising fp16.
* [TTJ] ttj.kr, "Huawei's KVarN - taming the KV cache with quantization",
  section "Dieting the cache with quantization": the engine keeps the KV
  cache in fixed-size pages (PagedAttention).
* [NAR] narnarhi.com, "SwiftKV ...", main part 2: fixed-size pages with a
  logical -> physical mapping.

The pages fix the method only in outline.  The concrete definitions this
oracle follows (and the CUDA path implements independently, at d = 128; the
format functions below also define d = 64 and 256, for which the library
has no kernels yet) are:

1. Rotation: X' = X H with H the orthonormal Sylvester Hadamard matrix,
   H[j, k] = (-1)^popcount(j & k) / sqrt(d), natural order, no random signs.
2. Normalization, ``iters`` times, channel step first:
   sigma_j = max(std_i Y[i, j], eps); Y[:, j] /= sigma_j; C_j *= sigma_j
   rho_i   = max(std_j Y[i, j], eps); Y[i, :] /= rho_i;   R_i *= rho_i
   with std the centred population standard deviation (ddof 0), eps = 1e-6,
   C and R starting at one; after each iteration (C, R) -> (C / 2^k, R 2^k)
   with 2^k the power of two that puts max C in [1, 2) (Y unchanged).
3. Per-token asymmetric RTN: z_i = min_j Y, M_i = max_j Y,
   s_i = (M_i - z_i) / (2^b - 1), code = clamp(rne((Y - z_i) / s_i)), code 0
   where s_i == 0.
4. Stored metadata: s~ = fp16(s_i R_i), z~ = fp16(z_i R_i) per token and
   C~ = fp16(C_j) per channel, so that the dequantized rotated tile is
   X^'[i, j] = (code * s~_i + z~_i) * C~_j and the tile is X^ = X^' H
   (H is symmetric and its own inverse).
5. Decode: out = softmax(q K^T / sqrt(d)) V in fp64 over the dequantized
   tiles followed by the raw fp16 rows of the unfinished last tile.
6. Chunked prefill: each of a chunk's n query tokens attends, as in 5, to
   the cached context followed by the chunk's own raw fp16 rows up to and
   including itself (causal).

Variant (not on the pages; a randomized rotation): with a nonzero 32-bit
``seed`` the rotation is X' = X D_s H, D_s = diag(s) with s_j = -1 where the
j-th output of SplitMix64 started at state ``seed`` has its top bit set and
+1 otherwise (SplitMix64 as published by Steele, Lea and Flood, "Fast
splittable pseudorandom number generators", OOPSLA 2014: the state advances
by the golden-ratio gamma 0x9E3779B97F4A7C15 and each output is the state
passed through the finalizer z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31).  The inverse is
X = X' H D_s.  Seed 0 is the plain rotation of 1.

Precision.  Everything runs in fp64 unless a caller asks for float32: where a
floating-point value decides an integer code, the parity tests run the
quantizer in float32, the precision the GPU takes that decision in.

Every function below is pinned by ``tests/test_oracle_pins.py`` against
something other than itself (a library routine, a closed form, an invariant
or brute force); nothing here is "parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np

EPS = 1e-6          # std clamp of the normalization (both steps)
HEAD_DIM = 128      # d: the head size the library implements (the format below also defines d = 64, 256)
HEAD_DIMS = (64, 128, 256)
PAGE_TOKENS = 16    # P: tokens per page (block)


# ---------------------------------------------------------------------------
# Step 1: Hadamard rotation along the channels  [AXB, four-step paragraph]
# ---------------------------------------------------------------------------

def sylvester_hadamard(d: int, dtype=np.float64) -> np.ndarray:
    """Orthonormal Sylvester Hadamard matrix of order d (a power of two).

    Built by the Kronecker recursion H_{2m} = [[H_m, H_m], [H_m, -H_m]] and
    scaled by 1/sqrt(d), so H @ H = I and H is symmetric.
    """
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return (h / math.sqrt(d)).astype(dtype)


def sylvester_signs(d: int) -> np.ndarray:
    """The unnormalized +-1 Sylvester matrix (sqrt(d) times ``sylvester_hadamard``)."""
    return np.rint(sylvester_hadamard(d) * math.sqrt(d))


_MASK64 = (1 << 64) - 1


def splitmix64_outputs(seed: int, n: int) -> list:
    """The first n outputs of SplitMix64 started at state ``seed`` (the
    generator's published definition, restated in the module docstring)."""
    state = seed & _MASK64
    out = []
    for _ in range(n):
        state = (state + 0x9E3779B97F4A7C15) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        out.append(z ^ (z >> 31))
    return out


def rotation_signs(d: int, seed: int = 0) -> np.ndarray:
    """Channel signs s of the randomized rotation (all +1 for seed 0)."""
    if seed == 0:
        return np.ones(d, dtype=np.float64)
    return np.array([-1.0 if v >> 63 else 1.0 for v in splitmix64_outputs(seed, d)], dtype=np.float64)


def rotate(x: np.ndarray, dtype=np.float64, seed: int = 0) -> np.ndarray:
    """X' = X D_s H for token rows X[..., d] (the rotation of step 1; D_s = I
    for seed 0).

    Computed as (X times the signs times the +-1 matrix) / sqrt(d): for fp16
    inputs the +-1 sums are exact in fp64, so a rotated channel that is zero
    in exact arithmetic comes out exactly zero.
    """
    x = np.asarray(x).astype(dtype)
    d = x.shape[-1]
    xs = x * rotation_signs(d, seed).astype(dtype)
    return (xs @ sylvester_signs(d).astype(dtype)) / dtype(math.sqrt(d))


# ---------------------------------------------------------------------------
# Step 2: Sinkhorn-like variance normalization  [AXB, four-step paragraph]
# ---------------------------------------------------------------------------

def sinkhorn_normalize(xr: np.ndarray, iters: int, eps: float = EPS):
    """Alternating channel / token std normalization of one rotated tile.

    ``xr`` is T x d.  Returns (Y, C, R): the normalized tile and the channel
    and token vectors accumulated multiplicatively, so that
    Y[i, j] * R[i] * C[j] == xr[i, j] up to rounding.

    (R, C) is only defined up to a common factor.  After every iteration the
    pair is rescaled by an exact power of two so that max_j C_j lies in
    [1, 2).  Y is untouched (bit for bit); without it the clamp makes C
    shrink like eps^n and R grow like eps^-n on degenerate tiles (a tile of
    identical tokens), and the fp16 metadata would overflow.
    """
    y = np.array(xr, copy=True)
    dt = y.dtype.type
    t, d = y.shape
    c = np.ones(d, dtype=y.dtype)
    r = np.ones(t, dtype=y.dtype)
    for _ in range(iters):
        # std is shift-invariant; taking it of the values minus the first
        # sample makes an exactly constant channel (or token) give exactly 0
        # in any precision, so the clamp decides as the definition says
        sigma = np.maximum((y - y[:1, :]).std(axis=0), dt(eps))   # each channel over the tile's tokens
        y = y / sigma[None, :]
        c = c * sigma
        rho = np.maximum((y - y[:, :1]).std(axis=1), dt(eps))     # each token over the channels
        y = y / rho[:, None]
        r = r * rho
        _, e = np.frexp(c.max())                        # max C = m 2^e, m in [0.5, 1)
        c = np.ldexp(c, 1 - int(e))
        r = np.ldexp(r, int(e) - 1)
    return y, c, r


# ---------------------------------------------------------------------------
# Step 3: per-token asymmetric round-to-nearest  [AXB, four-step paragraph]
# ---------------------------------------------------------------------------

def asymmetric_rtn(y: np.ndarray, bits: int):
    """Per-row asymmetric RTN of a T x d block.

    Returns (codes uint8 T x d, s T, z T) with zero = row min, scale =
    (max - min) / (2^b - 1) and round-half-to-even.
    """
    dt = y.dtype.type
    qmax = (1 << bits) - 1
    z = y.min(axis=1)
    m = y.max(axis=1)
    s = (m - z) / dt(qmax)
    codes = np.zeros(y.shape, dtype=np.uint8)
    live = s > 0
    if np.any(live):
        q = (y[live] - z[live, None]) / s[live, None]
        codes[live] = np.clip(np.rint(q), 0, qmax).astype(np.uint8)
    return codes, s, z


# ---------------------------------------------------------------------------
# The whole tile quantizer and its inverse
# ---------------------------------------------------------------------------

def quantize_tile(x: np.ndarray, bits: int, iters: int, eps: float = EPS,
                  dtype=np.float64, return_parts: bool = False, seed: int = 0):
    """Quantize one T x d tile of raw fp16 K or V rows (steps 1-4 above).

    Returns a dict with ``codes`` (uint8 T x d), ``s_t`` / ``z_t`` (fp16 per
    token, already multiplied by R) and ``c_t`` (fp16 per channel).  With
    ``return_parts`` it also carries the unrounded Y, s, z, C, R.
    """
    x = np.asarray(x)
    if x.ndim != 2:
        raise ValueError("a tile is T x d")
    xr = rotate(x.astype(np.float16).astype(dtype), dtype, seed)
    y, c, r = sinkhorn_normalize(xr, iters, eps)
    codes, s, z = asymmetric_rtn(y, bits)
    out = {
        "codes": codes,
        "s_t": (s * r).astype(np.float16),
        "z_t": (z * r).astype(np.float16),
        "c_t": c.astype(np.float16),
    }
    if return_parts:
        out.update(y=y, s=s, z=z, c=c, r=r, xr=xr)
    return out


def dequantize_tile(codes, s_t, z_t, c_t, seed: int = 0):
    """Inverse of ``quantize_tile`` in fp64.

    Returns (rotated-domain tile X^', original-domain tile X^ = X^' H D_s).
    """
    codes = np.asarray(codes, dtype=np.float64)
    s = np.asarray(s_t, dtype=np.float64)
    z = np.asarray(z_t, dtype=np.float64)
    c = np.asarray(c_t, dtype=np.float64)
    xr_hat = (codes * s[:, None] + z[:, None]) * c[None, :]
    d = codes.shape[1]
    return xr_hat, (xr_hat @ sylvester_hadamard(d)) * rotation_signs(d, seed)[None, :]


def plain_rtn_baseline(x: np.ndarray, bits: int) -> np.ndarray:
    """Plain per-token RTN of the raw tile (no rotation, no normalization),
    with fp16 scale and zero; returns the fp64 reconstruction."""
    x = np.asarray(x).astype(np.float16).astype(np.float64)
    codes, s, z = asymmetric_rtn(x, bits)
    s16 = s.astype(np.float16).astype(np.float64)
    z16 = z.astype(np.float16).astype(np.float64)
    return codes * s16[:, None] + z16[:, None]


# ---------------------------------------------------------------------------
# Page format (the layout written in include/kvq.h, restated here)
# ---------------------------------------------------------------------------

def page_layout(bits: int, tile_tokens: int, d: int = HEAD_DIM, p: int = PAGE_TOKENS):
    """Byte sizes / offsets of one page region of one KV head.

    codes (p*d*bits/8 bytes) | meta: p x {fp16 s~, fp16 z~} | C slice: fp16
    of the d*p/T channels this page of its tile carries.  Every region
    starts on a 16-byte boundary.
    """
    if tile_tokens % p or (d * p) % tile_tokens:
        raise ValueError("T must be a multiple of P and divide d*P")
    def up16(n):
        return (n + 15) // 16 * 16
    codes = up16(p * d * bits // 8)
    meta = up16(4 * p)
    cslice_ch = d * p // tile_tokens
    cslice = up16(2 * cslice_ch)
    return {"codes": codes, "meta_off": codes, "cslice_off": codes + meta,
            "cslice_channels": cslice_ch, "page_bytes": codes + meta + cslice}


def code_bit_position(channel: int, token: int, bits: int, is_v: bool,
                      d: int = HEAD_DIM) -> int:
    """Bit offset, inside a page's codes region, of the code of (channel,
    token-in-page).

    K (and V at 3 bits): a plain little-endian bitstream, token-major:
    field index token * d + channel.

    V at 2, 4 or 8 bits: grouped for the decode kernel's register layout.
    n = channel // 8 and g = channel % 8; t = (token % 8) // 2,
    u = token // 8 and s = token % 2.  The page's 32 "lanes" are
    L = 4 g + t.  Each lane owns W = d*bits/64 little-endian 32-bit words
    (2*bits at d = 128) holding the codes of its d/8 channels (n = 0..d/8-1)
    for the token pairs {2t, 2t+1} (u = 0) and {2t+8, 2t+9} (u = 1).  With
    F = 32 / bits fields per word and h = F / 2 pairs per word, the code
    lives in word k = 2 (n // h) + u at field e + h s, e = n % h.  Lane L's
    words sit in rows of R = min(4, W) words: word k is at byte
    ((k // R) * 32 + L) * 4R + (k % R) * 4 (R = 4 for every b at d >= 128;
    R = 2 only at d = 64, b = 2).
    """
    if not is_v or bits == 3:
        return (token * d + channel) * bits
    if d not in HEAD_DIMS or bits not in (2, 4, 8):
        raise ValueError("grouped V layout is defined for d in {64, 128, 256}, b in {2, 4, 8}")
    n, g = divmod(channel, 8)
    t = (token % 8) // 2
    u = token // 8
    s = token % 2
    fields_per_word = 32 // bits
    h = fields_per_word // 2
    k = 2 * (n // h) + u
    e = n % h
    lane = 4 * g + t
    row = min(4, d * bits // 64)  # words per lane row
    word_byte = ((k // row) * 32 + lane) * (4 * row) + (k % row) * 4
    return word_byte * 8 + bits * (e + h * s)


def pack_page_codes(codes_page: np.ndarray, bits: int, is_v: bool) -> np.ndarray:
    """Pack a P x d array of codes (token, channel) into the codes region."""
    p, d = codes_page.shape
    nbytes = p * d * bits // 8
    out = np.zeros(nbytes, dtype=np.uint8)
    for tok in range(p):
        for ch in range(d):
            val = int(codes_page[tok, ch])
            pos = code_bit_position(ch, tok, bits, is_v, d)
            for bit in range(bits):
                if (val >> bit) & 1:
                    q = pos + bit
                    out[q >> 3] |= np.uint8(1 << (q & 7))
    return out


def unpack_page_codes(region: np.ndarray, bits: int, is_v: bool,
                      p: int = PAGE_TOKENS, d: int = HEAD_DIM) -> np.ndarray:
    """Inverse of ``pack_page_codes``."""
    region = np.asarray(region, dtype=np.uint8)
    out = np.zeros((p, d), dtype=np.uint8)
    for tok in range(p):
        for ch in range(d):
            pos = code_bit_position(ch, tok, bits, is_v, d)
            val = 0
            for bit in range(bits):
                q = pos + bit
                val |= ((int(region[q >> 3]) >> (q & 7)) & 1) << bit
            out[tok, ch] = val
    return out


def write_tile_pages(pool: np.ndarray, block_ids, head: int, tile: dict,
                     bits: int, tile_tokens: int, is_v: bool) -> None:
    """Store one quantized tile into its T/P pages of a pool shaped
    [num_blocks][H_kv][page_bytes] (uint8).  ``block_ids`` are the physical
    blocks of the tile's pages in order."""
    d = tile["codes"].shape[1]
    lay = page_layout(bits, tile_tokens, d)
    p = PAGE_TOKENS
    cs = lay["cslice_channels"]
    for k, blk in enumerate(block_ids):
        region = pool[blk, head]
        region[:] = 0
        toks = slice(k * p, (k + 1) * p)
        region[:p * d * bits // 8] = pack_page_codes(tile["codes"][toks], bits, is_v)
        meta = np.stack([tile["s_t"][toks], tile["z_t"][toks]], axis=1).astype(np.float16)
        region[lay["meta_off"]:lay["meta_off"] + 4 * p] = meta.reshape(-1).view(np.uint8)
        cvals = tile["c_t"][k * cs:(k + 1) * cs].astype(np.float16)
        region[lay["cslice_off"]:lay["cslice_off"] + 2 * cs] = cvals.view(np.uint8)


def read_tile_pages(pool: np.ndarray, block_ids, head: int, bits: int,
                    tile_tokens: int, is_v: bool, d: int = HEAD_DIM) -> dict:
    """Inverse of ``write_tile_pages`` (used on pages the oracle packed)."""
    lay = page_layout(bits, tile_tokens, d)
    p = PAGE_TOKENS
    cs = lay["cslice_channels"]
    codes, s_t, z_t, c_t = [], [], [], []
    for blk in block_ids:
        region = np.asarray(pool[blk, head], dtype=np.uint8)
        codes.append(unpack_page_codes(region[:p * d * bits // 8], bits, is_v, d=d))
        meta = region[lay["meta_off"]:lay["meta_off"] + 4 * p].copy().view(np.float16).reshape(p, 2)
        s_t.append(meta[:, 0])
        z_t.append(meta[:, 1])
        c_t.append(region[lay["cslice_off"]:lay["cslice_off"] + 2 * cs].copy().view(np.float16))
    return {"codes": np.concatenate(codes), "s_t": np.concatenate(s_t),
            "z_t": np.concatenate(z_t), "c_t": np.concatenate(c_t)}


# ---------------------------------------------------------------------------
# Decode over the paged cache  [AIT, TL;DR]
# ---------------------------------------------------------------------------

def attention_fp64(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float | None = None):
    """softmax(q k^T * scale) v for one query head: q [d], k, v [L][d]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    logits = (k @ q) * scale
    logits -= logits.max()
    w = np.exp(logits)
    return (w[:, None] * v).sum(axis=0) / w.sum()


def sequence_kv_hat(tiles, tail_rows: np.ndarray, seed: int = 0) -> np.ndarray:
    """Original-domain K^ (or V^) of one (sequence, KV head): the
    dequantized full tiles in order, then the raw fp16 rows of the unfinished
    tile.  ``tiles`` is a list of ``quantize_tile``-style dicts."""
    parts = [dequantize_tile(t["codes"], t["s_t"], t["z_t"], t["c_t"], seed)[1] for t in tiles]
    d = tiles[0]["codes"].shape[1] if tiles else np.asarray(tail_rows).shape[-1]
    parts.append(np.asarray(tail_rows, dtype=np.float16).astype(np.float64).reshape(-1, d))
    return np.concatenate(parts, axis=0)


def decode_sequence(q_heads: np.ndarray, k_hat: list, v_hat: list, group: int,
                    scale: float | None = None) -> np.ndarray:
    """Decode one sequence: q_heads [H_q][d]; k_hat / v_hat lists indexed by KV
    head of [L][d] arrays; query head h reads KV head h // group."""
    out = np.zeros(q_heads.shape, dtype=np.float64)
    for h in range(q_heads.shape[0]):
        out[h] = attention_fp64(q_heads[h], k_hat[h // group], v_hat[h // group], scale)
    return out


def prefill_chunk_sequence(q_chunk: np.ndarray, k_hat: list, v_hat: list, k_new: np.ndarray,
                           v_new: np.ndarray, group: int, scale: float | None = None) -> np.ndarray:
    """Chunked prefill of one sequence over its cache  [AIT, TL;DR].

    The attention backend reads the compressed pages in every phase, so a
    chunk of n new tokens attends to the cached context as stored (the
    dequantized tiles, then the raw tail: ``k_hat`` / ``v_hat``, lists
    indexed by KV head of [L][d]) and to the chunk's own rows, which are not
    in the cache yet and enter as the raw fp16 rows they are.  Chunk token i
    sees the L context tokens and chunk tokens 0..i (causal); query head h
    reads KV head h // group.

    q_chunk [n][H_q][d]; k_new / v_new [n][H_kv][d].  Returns [n][H_q][d]
    (fp64).  Appending the chunk to the cache afterwards is the write path's
    business (tiles the chunk completes get quantized), not this function's.
    """
    q_chunk = np.asarray(q_chunk, dtype=np.float64)
    k_new = np.asarray(k_new, dtype=np.float16).astype(np.float64)
    v_new = np.asarray(v_new, dtype=np.float16).astype(np.float64)
    n, hq = q_chunk.shape[:2]
    out = np.zeros(q_chunk.shape, dtype=np.float64)
    for i in range(n):
        for h in range(hq):
            kv = h // group
            keys = np.concatenate([k_hat[kv], k_new[:i + 1, kv]], axis=0)
            vals = np.concatenate([v_hat[kv], v_new[:i + 1, kv]], axis=0)
            out[i, h] = attention_fp64(q_chunk[i, h], keys, vals, scale)
    return out


def quantize_sequence(rows: np.ndarray, tile_tokens: int, bits: int, iters: int,
                      dtype=np.float64, seed: int = 0):
    """Quantize every full tile of one (sequence, KV head): rows [L][d] fp16.
    Returns (list of tile dicts, raw tail rows)."""
    n_full = rows.shape[0] // tile_tokens
    tiles = [quantize_tile(rows[t * tile_tokens:(t + 1) * tile_tokens], bits, iters, dtype=dtype, seed=seed)
             for t in range(n_full)]
    return tiles, rows[n_full * tile_tokens:]
