/*
 * kvq.h - C ABI of the B200 (sm_100a) quantized paged KV-cache library.
 *
 * What the library computes
 * -------------------------
 * The method is the one described on axbrief.com, "Huawei's KVarN boosts
 * vLLM KV-cache capacity by 5x without accuracy loss", section "What
 * differs from existing methods" (the four-step paragraph): the fp16 K/V
 * cache is quantized in fixed-size token tiles; each tile gets a Hadamard
 * rotation along the head-dim channels, then Sinkhorn-like alternating
 * channel / token variance normalization, then asymmetric round-to-nearest
 * to b-bit codes.  Attention reads the packed pages directly (aitrends.kr
 * article 74976, "TL;DR" and glossary "attention backend"); pages follow
 * PagedAttention's fixed-size blocks with a logical -> physical block table
 * (ttj.kr KVarN explainer, "Dieting the cache with quantization";
 * narnarhi.com "SwiftKV ...", main part 2).
 *
 * Definitions (the pages give the outline only; these are the concrete
 * readings the library implements):
 *   d = head_dim in {64,128,256}, P = page_tokens = 16, T = tile_tokens in {32,64,128},
 *   b = bits in {2,3,4,8} (8 for K and V together), n = iters >= 0,
 *   eps = std_eps (1e-6).
 *   H = orthonormal Sylvester Hadamard, H[j][k] = (-1)^popcount(j&k)/sqrt(d).
 *   For one tile X (T x d fp16, one sequence, one KV head, K or V):
 *     Y = X H;  C = 1_d;  R = 1_T;  repeat n times:
 *       sigma_j = max(std_i Y_ij, eps);  Y_:j /= sigma_j;  C_j *= sigma_j
 *       rho_i   = max(std_j Y_ij, eps);  Y_i: /= rho_i;    R_i *= rho_i
 *       (C, R) <- (C / 2^k, R * 2^k), 2^k the power of two with max C in [1,2)
 *     std = centred population standard deviation (ddof 0).
 *     Per token i: z_i = min_j Y_ij, s_i = (max_j Y_ij - z_i) / (2^b - 1),
 *     code_ij = clamp(round_half_even((Y_ij - z_i) / s_i), 0, 2^b - 1)
 *     (all codes 0 when s_i == 0).
 *     Stored: s~_i = fp16(s_i R_i), z~_i = fp16(z_i R_i), C~_j = fp16(C_j).
 *   Dequantization: X^'_ij = (code_ij s~_i + z~_i) C~_j and X^ = X^' H.
 *   Randomized rotation (a variant, not on the pages): with rotation_seed
 *   != 0 every H above becomes D_s H on the way in (Y = X D_s H, q' = H D_s q)
 *   and H D_s on the way out (X^ = X^' H D_s, out = D_s H acc'), D_s =
 *   diag(s) with s_j = -1 where the j-th output (j = 0..d-1) of SplitMix64
 *   started at state rotation_seed has its top bit set, else +1.  SplitMix64
 *   (Steele, Lea and Flood, OOPSLA 2014): state += 0x9E3779B97F4A7C15;
 *   z = state; z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9;
 *   z = (z ^ (z >> 27)) * 0x94D049BB133111EB; output z ^ (z >> 31).
 *   A sequence of L tokens holds floor(L/T) quantized tiles, tile t covering
 *   tokens [tT, (t+1)T); the last L mod T tokens stay raw fp16 in a tail
 *   buffer until their tile fills.
 *   Decode: out_h = softmax(q_h K^T * scale) V over the dequantized tiles and
 *   the raw tail of KV head h / g, computed as: q' = H q (once), scores and
 *   P V on the packed codes in the rotated domain, one inverse rotation H of
 *   the accumulated output, plus the raw-domain tail; split-K over tiles
 *   with a log-sum-exp merge.
 *
 * Page format (version 1)
 * -----------------------
 *   K pool and V pool are separate device buffers, each
 *     uint8 pool[num_blocks][num_kv_heads][page_bytes]
 *   One page region (block, head) holds P tokens of one KV head:
 *     [codes | meta | C slice], each region starting on a 16-byte boundary.
 *   codes: P*d*b/8 bytes (at d=128: 2048 at b=8, 1024 at b=4, 768 at b=3, 512 at b=2), a little-
 *     endian bitstream; a code occupies b bits at the bit offset below.
 *   meta:  P entries of {fp16 s~, fp16 z~} (64 bytes), token-major.
 *   C slice: page k of its tile (k = logical block index mod T/P) carries
 *     fp16 C~ of channels [k*d*P/T, (k+1)*d*P/T)  (2*d*P/T bytes).
 *   page_bytes = codes + 64 + 2*d*P/T rounded up to 16  (1152 for d=128, T=64, b=4).
 *   Bit offset of the code of (channel c, token p of the page):
 *     K, and V at b=3:   (p*d + c) * b                (token-major)
 *     V at b in {2,4,8}: the decode kernel's grouped order.  With
 *       n = c/8, g = c%8, t = (p%8)/2, u = p/8, s = p%2, F = 32/b,
 *       h = F/2, k = 2*(n/h) + u, e = n%h, lane = 4*g + t, W = d*b/64
 *       words per lane in rows of R = min(4, W) words (R = 4 except d=64, b=2):
 *       byte of word = ((k/R)*32 + lane)*4R + (k%R)*4,
 *       bit offset   = 8*(byte of word) + b*(e + h*s).
 *   Tails: fp16 [num_seqs][num_kv_heads][T][d], one for K and one for V;
 *     token position q of a sequence lives in row q mod T.
 *   Query / output: fp16 [num_seqs][num_kv_heads*group_size][d]; query head
 *     h reads KV head h / group_size.
 *
 * Head sizes
 * ----------
 *   d = 128 runs the tuned path (tensor-core rotation in the quantizer,
 *   mma.sync decode, tensor-core chunked prefill, the one-launch serving
 *   step).  d = 64 and d = 256 run every call on CUDA-core kernels with the
 *   same format, the same method and the same contracts, with two
 *   differences: chunked prefill runs one launch over the whole context and
 *   needs no workspace (kvq_prefill_workspace_bytes gives 0 for every
 *   num_splits, which is checked and otherwise ignored), and
 *   kvq_append_decode_step runs as three launches (the tokens into the tails
 *   and the lengths advanced, then the split-K decode and its merge).
 *
 * Conventions
 * -----------
 *  - Every pointer argument marked "device" is a device pointer of the
 *    current CUDA device; every such pointer must be 16-byte aligned.
 *  - The caller owns every buffer (pools, tails, tables, workspace, status
 *    word).  No call allocates device memory.  State kept by the library:
 *    a thread-local error message, and for
 *    kvq_paged_decode_attention_static_scratch a static device array of
 *    KVQ_DECODE_STATIC_SCRATCH_BYTES (32 MiB) that is part of the library's
 *    device code, so every device that loads the library's module (at its
 *    first kernel launch, or at start-up with CUDA_MODULE_LOADING=EAGER)
 *    holds those 32 MiB until the process exits, whether or not that entry
 *    point is ever called; plus that array's address per device.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream) and
 *    never synchronizes.  Arguments are validated on the host first; an
 *    invalid call returns an error and launches nothing.
 *  - Errors the device detects (a block id outside [0, num_blocks), a
 *    missing page) are written once into *dev_status (device int32, may be
 *    NULL; the first error wins) and the affected work item is skipped.
 *    Nothing traps.  A launch failure returns KVQ_ERR_CUDA.
 *  - The caller allocates pages before appending and owns seq_lens.
 */
#ifndef KVQ_H_
#define KVQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,   /* bad pointer, size, or configuration value   */
  KVQ_ERR_UNSUPPORTED = 2,   /* valid but not implemented (e.g. d = 96)     */
  KVQ_ERR_CUDA = 3,          /* a CUDA runtime call or launch failed        */
  KVQ_ERR_WORKSPACE = 4,     /* decode workspace smaller than required      */
  KVQ_ERR_DEVICE_BOUNDS = 5, /* device saw a block id out of range          */
  KVQ_ERR_DEVICE_TIMEOUT = 6 /* a bounded device wait gave up               */
} kvq_status;

typedef struct {
  int head_dim;      /* d: 64, 128 or 256 (see the head-size note)       */
  int num_kv_heads;  /* H_kv >= 1                                        */
  int group_size;    /* g = query heads per KV head, 1..8                */
  int tile_tokens;   /* T: 32, 64 or 128                                 */
  int page_tokens;   /* P: must be 16                                    */
  int bits_k;        /* b for K codes: 2, 3, 4 or 8 (8 with bits_v = 8) */
  int bits_v;        /* b for V codes: 2, 3, 4 or 8 (8 with bits_k = 8) */
  int iters;         /* n: normalization iterations, 0..64               */
  float std_eps;     /* std clamp, > 0 (1e-6 in the method)              */
  uint32_t rotation_seed; /* 0: the rotation H; else the randomized       */
                          /* rotation D_s H (see Definitions)             */
} kvq_config;

typedef struct {
  size_t page_bytes_k, page_bytes_v;     /* one (block, head) page region   */
  size_t codes_bytes_k, codes_bytes_v;   /* codes region = meta offset      */
  size_t cslice_off_k, cslice_off_v;     /* C-slice offset in the region    */
  size_t block_stride_k, block_stride_v; /* num_kv_heads * page_bytes       */
  size_t tail_bytes;                     /* one tail buffer (K or V) per sequence:
                                            num_kv_heads * T * d * 2        */
  int cslice_channels;                   /* d * P / T                       */
  int pages_per_tile;                    /* T / P                           */
} kvq_layout;

/* Fill *out with the byte layout of config *cfg.
 * cfg, out: host pointers.  Returns KVQ_ERR_INVALID_ARG for a bad config. */
KVQ_API kvq_status kvq_get_layout(const kvq_config* cfg, kvq_layout* out);

/* Bytes of device workspace kvq_paged_decode_attention needs for num_seqs
 * sequences and num_splits (0 = automatic) on the current device.
 * cfg, bytes: host pointers. */
KVQ_API kvq_status kvq_decode_workspace_bytes(const kvq_config* cfg, int num_seqs, int num_splits,
                                      size_t* bytes);

/* Write path, prefill: quantize full tiles of raw rows into the pools.
 *   src_k, src_v : device fp16 [num_rows][num_kv_heads][d]; either may be NULL
 *                  to skip K or V.
 *   tile_desc    : device int32 [num_tiles][3] = {src_row, seq, tile_idx}:
 *                  tile tokens are rows src_row .. src_row+T-1 and land in the
 *                  pages of logical blocks tile_idx*T/P .. +T/P-1 of seq.
 *   block_tables : device int32 [num_seqs][max_blocks_per_seq].
 *   k_pool/v_pool: device uint8 pools (layout above).
 * Every KV head of every listed tile is quantized (one work item per tile,
 * head and K/V).  A descriptor with rows outside [0, num_rows), a sequence
 * outside [0, num_seqs) or pages outside the table is skipped and reported
 * through dev_status (KVQ_ERR_DEVICE_BOUNDS). */
KVQ_API kvq_status kvq_quantize_tiles(const kvq_config* cfg, const void* src_k, const void* src_v,
                              int num_rows, const int32_t* tile_desc, int num_tiles,
                              const int32_t* block_tables, int num_seqs, int max_blocks_per_seq,
                              int num_blocks, void* k_pool, void* v_pool,
                              int32_t* dev_status, void* stream);

/* Write path, decode / chunked prefill: append new tokens.
 *   new_k, new_v     : device fp16 [cu_new[num_seqs]][num_kv_heads][d].
 *   cu_new           : device int32 [num_seqs+1], prefix sums of new tokens.
 *   seq_lens_before  : device int32 [num_seqs], tokens already cached.
 *   max_new_per_seq  : host bound on cu_new[s+1]-cu_new[s] (>= 0).
 *   k_tail, v_tail   : device fp16 tails [num_seqs][num_kv_heads][T][d].
 * Every tile completed by the new tokens is quantized (from the old tail
 * rows and the new rows) into its pages; the remaining new tokens land in
 * the tail.  The result is bit-identical to kvq_quantize_tiles on the same
 * tokens.  seq_lens is not updated (the caller owns it). */
KVQ_API kvq_status kvq_append_tokens(const kvq_config* cfg, const void* new_k, const void* new_v,
                             const int32_t* cu_new, const int32_t* seq_lens_before,
                             int num_seqs, int max_new_per_seq,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             int num_blocks, void* k_pool, void* v_pool,
                             void* k_tail, void* v_tail, int32_t* dev_status, void* stream);

/* Read path: one decode step of paged attention over the quantized cache.
 *   q, out       : device fp16 [num_seqs][num_kv_heads*group_size][d]; q is
 *                  not rotated (the kernel rotates it).
 *   seq_lens     : device int32 [num_seqs], tokens in the cache (including
 *                  any token appended for this step); full tiles come from
 *                  the pools, the last seq_len mod T tokens from the tails.
 *   softmax_scale: scale of q.k (1/sqrt(d) in the method).
 *   workspace    : device, >= kvq_decode_workspace_bytes(cfg, num_seqs,
 *                  num_splits) bytes; contents on entry are ignored.
 *   num_splits   : split-K factor over tiles per (sequence, KV head); 0 picks
 *                  one from the device size.  The output does not depend on it
 *                  beyond rounding.
 * Decode reads b in {2, 3, 4} for K and V (any combination), and 8 for
 * both.  3-bit pages are read code by code (their V layout is a plain
 * bitstream), so a 3-bit decode costs more instructions per byte than the
 * 2- and 4-bit ones. */
KVQ_API kvq_status kvq_paged_decode_attention(const kvq_config* cfg, const void* q, void* out,
                                      const int32_t* seq_lens, int num_seqs,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      int num_blocks, const void* k_pool, const void* v_pool,
                                      const void* k_tail, const void* v_tail,
                                      float softmax_scale, void* workspace,
                                      size_t workspace_bytes, int num_splits,
                                      int32_t* dev_status, void* stream);

/* One serving step in one launch (d = 128; three at d = 64 / 256): append one
 * token per sequence and decode.
 * The pages say the per-step read path decides the serving gain (aitrends.kr
 * article 74976, "TL;DR"); this call folds the step's append into the
 * decode launch, for steps in which no sequence completes a tile.
 *   new_k, new_v : device fp16 [num_seqs][num_kv_heads][d], the step's token
 *                  of every sequence.
 *   seq_lens     : device int32 [num_seqs], tokens cached BEFORE the step;
 *                  the call advances every entry by one when it finishes.
 *   q, out       : as kvq_paged_decode_attention (attention over the cache
 *                  including the step's token).
 *   k_tail, v_tail: device fp16 tails; the token goes to row seq_len mod T.
 *   num_splits   : 1..65535 chunks per (sequence, KV head), fixed (no
 *                  schedule launch); units past a short sequence's tiles are
 *                  empty.
 *   workspace    : device, >= kvq_decode_workspace_bytes(cfg, num_seqs,
 *                  num_splits) bytes, ZERO-FILLED before its first use (for
 *                  example cudaMemset at allocation).  Every call that
 *                  completes leaves its counters at zero again, so the same
 *                  workspace serves the next step without a clear; after a
 *                  call that reported a device error, zero it again.  Do not
 *                  share it with kvq_paged_decode_attention calls.
 * The result (out, tails, seq_lens) equals kvq_append_tokens of the same
 * rows, the lengths advanced by one, then kvq_paged_decode_attention with the
 * same num_splits (bit for bit).  Precondition: no sequence's token completes
 * a tile (seq_len + 1 is not a multiple of T); such a token has to be
 * quantized into pages, which this launch does not do: it is not written,
 * KVQ_ERR_DEVICE_BOUNDS is reported, and that sequence's output is not
 * valid.  Use kvq_append_tokens then kvq_paged_decode_attention for those
 * steps.  Host-side errors as kvq_paged_decode_attention; the call is
 * asynchronous on stream. */
KVQ_API kvq_status kvq_append_decode_step(const kvq_config* cfg, const void* new_k, const void* new_v,
                                          const void* q, void* out, int32_t* seq_lens, int num_seqs,
                                          const int32_t* block_tables, int max_blocks_per_seq, int num_blocks,
                                          const void* k_pool, const void* v_pool, void* k_tail, void* v_tail,
                                          float softmax_scale, void* workspace, size_t workspace_bytes,
                                          int num_splits, int32_t* dev_status, void* stream);

/* Bytes of device workspace kvq_paged_prefill_attention needs with num_splits
 * context splits (0 for num_splits = 1, and 0 at d = 64 / 256).  cfg, bytes:
 * host pointers. */
KVQ_API kvq_status kvq_prefill_workspace_bytes(const kvq_config* cfg, int num_seqs, int max_chunk_tokens,
                                               int num_splits, size_t* bytes);

/* Read path, chunked prefill: attention of a chunk of new tokens per sequence
 * over the quantized cache and the chunk itself.  The method reads the
 * compressed pages directly in every phase of attention (aitrends.kr article
 * 74976, "TL;DR"; glossary "attention backend"); the chunk's own rows are not
 * cached yet and enter as raw fp16.  Chunk token i of sequence s (query head
 * j, reading KV head j / group_size) attends to the ctx_lens[s] cached tokens
 * (full tiles from the pools, the last ctx_lens[s] mod T from the tails) and
 * to chunk tokens 0..i: softmax(q.k * softmax_scale) V in fp32.
 *   q, out       : device fp16 [cu_chunk[num_seqs]][num_kv_heads*group_size][d],
 *                  the chunk tokens of all sequences packed; q not rotated.
 *   k_new, v_new : device fp16 [cu_chunk[num_seqs]][num_kv_heads][d], the
 *                  chunk's K and V rows.
 *   cu_chunk     : device int32 [num_seqs+1], prefix sums of chunk lengths.
 *   ctx_lens     : device int32 [num_seqs], tokens cached before the chunk.
 *   max_chunk_tokens: host bound >= every chunk length (sizes the launch:
 *                  one CTA per sequence, KV head and 128 query rows, times
 *                  num_splits).
 *   num_splits   : 1..64.  1: one launch, each CTA runs its whole context.
 *                  S > 1: the context tiles of each (sequence, KV head, row
 *                  tile) are split over S CTAs that write partial softmax
 *                  states to the workspace, then a second launch merges them
 *                  (log-sum-exp) and adds the tail and the chunk rows; the
 *                  result does not depend on S beyond rounding.  More CTAs
 *                  fill the device when (sequences x KV heads x row tiles) is
 *                  small or leaves a partial last wave.
 *   workspace    : device, >= kvq_prefill_workspace_bytes(cfg, num_seqs,
 *                  max_chunk_tokens, num_splits) bytes (may be NULL when that
 *                  is 0); contents on entry are ignored.
 *   block_tables, k_pool, v_pool, k_tail, v_tail, num_blocks: the cache, as
 *                  for kvq_paged_decode_attention.
 *   softmax_scale: scale of q.k (1/sqrt(d) in the method).
 *   dev_status   : device int32, may be NULL; first device-detected error.
 *   stream       : cudaStream_t (NULL = legacy default stream); the call is
 *                  asynchronous on it.
 * All buffers are caller-owned device memory, 16-byte aligned; the library
 * keeps no pointer after the call.  Host-side checks (config, NULL or
 * misaligned pointers, num_seqs outside 0..65535, max_chunk_tokens outside
 * 0..2^20, num_splits outside 1..64, a non-positive or non-finite scale)
 * return KVQ_ERR_INVALID_ARG / KVQ_ERR_UNSUPPORTED, a short workspace
 * KVQ_ERR_WORKSPACE, before any launch.
 * The chunk is not appended: call kvq_append_tokens with the same rows and
 * cu_chunk afterwards (tiles it completes are then quantized).  A chunk
 * longer than max_chunk_tokens, or negative, is reported through dev_status
 * (KVQ_ERR_DEVICE_BOUNDS) and only its first max_chunk_tokens tokens are
 * written; pages outside the pool likewise (the tile is skipped).  b in
 * {2, 3, 4} for K and V (any combination), or 8 for both. */
KVQ_API kvq_status kvq_paged_prefill_attention(const kvq_config* cfg, const void* q, void* out,
                                       const void* k_new, const void* v_new, const int32_t* cu_chunk,
                                       const int32_t* ctx_lens, int num_seqs, int max_chunk_tokens,
                                       const int32_t* block_tables, int max_blocks_per_seq,
                                       int num_blocks, const void* k_pool, const void* v_pool,
                                       const void* k_tail, const void* v_tail, float softmax_scale,
                                       int num_splits, void* workspace, size_t workspace_bytes,
                                       int32_t* dev_status, void* stream);

/* Size of the scratch array built into the library for
 * kvq_paged_decode_attention_static_scratch (32 MiB per device). */
#define KVQ_DECODE_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

/* kvq_paged_decode_attention without a caller workspace.  The method on the
 * pages has no counterpart of this call: it exists for callers that cannot
 * allocate device memory when they decode (a runtime that gave the whole
 * device to its KV pool and weights at start-up, a serving loop that must not
 * take cudaMalloc's implicit device synchronization, a C embedding with no
 * device allocator).  It allocates and frees nothing.
 *   Arguments, layouts and results: as kvq_paged_decode_attention, minus
 *   workspace / workspace_bytes.  The workspace is a static device array of
 *   KVQ_DECODE_STATIC_SCRATCH_BYTES in the library, one per device.
 *   Size limit: if kvq_decode_workspace_bytes(cfg, num_seqs, num_splits)
 *   exceeds KVQ_DECODE_STATIC_SCRATCH_BYTES the call returns
 *   KVQ_ERR_WORKSPACE (detail in kvq_last_error) before touching the device;
 *   use fewer sequences per call, a smaller num_splits, or the workspace entry.
 *   Set-up: the first call on each device (that device current) looks up the
 *   array's address with cudaGetSymbolAddress and keeps it; make that first
 *   call before any stream capture begins.  Device ordinals 0..63.  The kept
 *   address belongs to the device's current context: after cudaDeviceReset
 *   (or any destruction of the primary context) the array may move, so do not
 *   call this entry point again in that process after a reset.
 *   Memory: the array is reserved on every device that loads the library's
 *   module, whether or not this entry point is called.
 *   Concurrency: calls on the same device share the array; two calls that
 *   overlap in time (different streams, or unordered host threads) race on it
 *   and corrupt each other's results.  Order them (one stream, or events). */
KVQ_API kvq_status kvq_paged_decode_attention_static_scratch(
    const kvq_config* cfg, const void* q, void* out, const int32_t* seq_lens, int num_seqs,
    const int32_t* block_tables, int max_blocks_per_seq, int num_blocks, const void* k_pool, const void* v_pool,
    const void* k_tail, const void* v_tail, float softmax_scale, int num_splits, int32_t* dev_status,
    void* stream);

/* Inspection (tests, tools): read num_tiles tiles back out of a pool.
 *   tile_desc : device int32 [num_tiles][2] = {seq, tile_idx}; all heads.
 *   is_v      : 0 = K pool / bits_k, 1 = V pool / bits_v.
 *   codes     : device uint8 [num_tiles][num_kv_heads][T][d]      (may be NULL)
 *   meta      : device fp16  [num_tiles][num_kv_heads][T][2] {s~, z~} (may be NULL)
 *   cvec      : device fp16  [num_tiles][num_kv_heads][d]        (may be NULL)
 *   out_rot   : device fp32  [num_tiles][num_kv_heads][T][d] dequantized,
 *               rotated domain (X^')                             (may be NULL)
 *   out_orig  : device fp32, same shape, original domain (X^' H)  (may be NULL) */
KVQ_API kvq_status kvq_unpack_tiles(const kvq_config* cfg, const int32_t* tile_desc, int num_tiles,
                            const int32_t* block_tables, int num_seqs, int max_blocks_per_seq, int num_blocks,
                            const void* pool, int is_v, uint8_t* codes, void* meta, void* cvec,
                            float* out_rot, float* out_orig, int32_t* dev_status, void* stream);

/* Self-test of device-side failure detection: launches, on `stream`, one
 * single-thread kernel per kernel file that waits with that file's bounded
 * mbarrier wait on a barrier nothing ever arrives at.  Each wait gives up
 * after its limit (2 s) and records KVQ_ERR_DEVICE_TIMEOUT in *dev_status
 * (device int32, required); nothing traps and the context stays usable.
 * Three such waits (quantize, decode, prefill kernels): about 6 s of device
 * time.  Returns KVQ_ERR_INVALID_ARG for a NULL
 * dev_status, KVQ_ERR_CUDA on a launch error. */
KVQ_API kvq_status kvq_selftest_bounded_wait(int32_t* dev_status, void* stream);

/* Static text for a status code. */
KVQ_API const char* kvq_status_string(kvq_status s);
/* Detail of the last error on the calling host thread ("" if none). */
KVQ_API const char* kvq_last_error(void);
/* Library version string ("kvq <major>.<minor> format 1 sm_100a"). */
KVQ_API const char* kvq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H_ */
