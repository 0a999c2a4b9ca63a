// Head sizes d = 64 and 256 on the CUDA cores: tile quantization (prefill and
// append with tile completion), paged decode attention, and the pool
// read-back.  The d = 128 path (tensor-core rotation, mma.sync decode) is in
// kvq_quantize_tc.cu and kvq_decode.cu; these kernels take the plainest route
// through the same method and the same page format at the other two head
// sizes, one CTA per tile (write path) or per (sequence, KV head, split)
// (read path), with the whole tile in shared memory.
//
// Method: axbrief.com "Huawei's KVarN boosts vLLM KV-cache capacity by 5x
// without accuracy loss", section "What differs from existing methods":
// per token tile, a Hadamard rotation along the head-dim channels,
// Sinkhorn-like alternating channel / token standard-deviation
// normalization, then per-token asymmetric round-to-nearest.  Read path:
// aitrends.kr article 74976, "TL;DR": attention reads the compressed pages
// directly, with the query rotated once and the output rotated back once.
//
// Rounding: the tile is fp32 and is divided by each std in turn, in the order
// the definition gives (IEEE division); the std sums accumulate in fp64.  For
// d = 64 and 256, 1/sqrt(d) is a power of two, so the scaling of the rotation
// is exact.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cfloat>
#include <cmath>

#include "kvq_device.cuh"

namespace kvq {

namespace {

constexpr int kGThreads = 256;
constexpr int kGWarps = kGThreads / 32;
constexpr int kMaxPages = 128 / kPageTokens;  // pages of the largest tile

// Bit offset of the code of (channel c, token p of the page) in a page's
// codes region, for head size D.  K, and V at 3 bits: a token-major
// little-endian bitstream.  V at 2, 4 and 8 bits: decode-lane groups, lane
// 4g + t owning W = D b / 64 words (channels 8n + g, token pairs {2t, 2t + 1}
// and {2t + 8, 2t + 9}) in rows of min(4, W) words.
template <int D>
__device__ __forceinline__ int code_bit_d(int c, int p, int bits, bool is_v) {
  if (!is_v || bits == 3) return (p * D + c) * bits;
  const int n = c >> 3, g = c & 7;
  const int t = (p & 7) >> 1, u = p >> 3, s = p & 1;
  const int h = 16 / bits;  // code pairs per 32-bit word
  const int k = 2 * (n / h) + u;
  const int e = n % h;
  const int lane = 4 * g + t;
  const int w = D * bits / 64;
  const int rw = w < 4 ? w : 4;
  const int word_byte = ((k / rw) * 32 + lane) * (4 * rw) + (k % rw) * 4;
  return word_byte * 8 + bits * (e + h * s);
}

// Set a b-bit code at `bit` in a zeroed run of 32-bit words (shared memory);
// a 3-bit field may straddle two words.
__device__ __forceinline__ void put_code(uint32_t* words, int bit, int bits, uint32_t code) {
  const int w = bit >> 5, sh = bit & 31;
  atomicOr(&words[w], code << sh);
  if (sh + bits > 32) atomicOr(&words[w + 1], code >> (32 - sh));
}

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}

__device__ __forceinline__ float block_max(float v, float* red) {
  v = warp_max(v);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
  for (int w = 1; w < kGWarps; ++w) m = fmaxf(m, red[w]);
  __syncthreads();
  return m;
}

// In-place Walsh-Hadamard transform (natural order, unnormalized) of `rows`
// rows of D floats at stride ld in shared memory, by the whole CTA.
template <int D>
__device__ void fwht_rows(float* y, int rows, int ld) {
  for (int h = 1; h < D; h <<= 1) {
    for (int idx = threadIdx.x; idx < rows * (D / 2); idx += kGThreads) {
      const int i = idx / (D / 2), k = idx % (D / 2);
      const int j = (k / h) * 2 * h + (k % h);
      float* row = y + i * ld;
      const float a = row[j], b = row[j + h];
      row[j] = a + b;
      row[j + h] = a - b;
    }
    __syncthreads();
  }
}

template <int D>
constexpr float inv_sqrt_d() {
  return D == 64 ? 0.125f : 0.0625f;  // 1/sqrt(64), 1/sqrt(256): exact powers of two
}

// Shared memory of the tile quantizer: Y [T][D + 1] floats, c [D], r [T],
// 32 floats of reduction space, then the staging copy of the tile's T/P pages.
template <int D>
__host__ __device__ constexpr size_t gq_stage_off(int T) {
  return (static_cast<size_t>(T) * (D + 1) + D + T + 32) * sizeof(float);
}
size_t gq_smem_bytes(int D, int T, int page_bytes) {
  const size_t off = (static_cast<size_t>(T) * (D + 1) + D + T + 32) * sizeof(float);
  return (off + 15) / 16 * 16 + static_cast<size_t>(T / kPageTokens) * page_bytes;
}

// One tile of one (KV head, K|V) by the whole CTA: rotation, normalization,
// RTN, packing, page stores.  row_of(i) gives the fp16 row of token i of the
// tile; blk[k] the block of page k (checked by the caller).
template <int D, class RowOf>
__device__ void quantize_tile_generic(const RowOf& row_of, int T, bool is_v, const kvq_config& cfg,
                                      const PoolGeom& g, const int* blk, uint8_t* pool, int head,
                                      unsigned char* smem) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int ld = D + 1;
  float* y = reinterpret_cast<float*>(smem);
  float* c = y + T * ld;
  float* r = c + D;
  float* red = r + T;
  unsigned char* stage = smem + (gq_stage_off<D>(T) + 15) / 16 * 16;
  const int npages = T / kPageTokens;
  const int bits = g.bits;
  const int qmax = (1 << bits) - 1;
  const float eps = cfg.std_eps;

  for (int i = tid; i < npages * g.page_bytes / 16; i += kGThreads)
    reinterpret_cast<uint4*>(stage)[i] = make_uint4(0u, 0u, 0u, 0u);
  // rows times the channel signs of the randomized rotation (all +1 for seed 0)
  for (int idx = tid; idx < T * D; idx += kGThreads) {
    const int i = idx / D, j = idx % D;
    y[i * ld + j] = __half2float(row_of(i)[j]) * rotation_sign(cfg.rotation_seed, j);
  }
  for (int j = tid; j < D; j += kGThreads) c[j] = 1.f;
  for (int i = tid; i < T; i += kGThreads) r[i] = 1.f;
  __syncthreads();
  fwht_rows<D>(y, T, ld);
  for (int idx = tid; idx < T * D; idx += kGThreads) y[(idx / D) * ld + idx % D] *= inv_sqrt_d<D>();
  __syncthreads();

  for (int it = 0; it < cfg.iters; ++it) {
    // channel step: std over the tile's tokens of (y - y[0][j]), clamped
    // (the sums in fp64: up to 256 terms, kept well inside the rounding-tie
    // band of the codes)
    for (int j = tid; j < D; j += kGThreads) {
      const double sh = y[j];
      double s1 = 0.0;
      for (int i = 0; i < T; ++i) s1 += static_cast<double>(y[i * ld + j]) - sh;
      const double mean = s1 / T;
      double s2 = 0.0;
      for (int i = 0; i < T; ++i) {
        const double dd = (static_cast<double>(y[i * ld + j]) - sh) - mean;
        s2 += dd * dd;
      }
      const float sigma = fmaxf(static_cast<float>(sqrt(s2 / T)), eps);
      for (int i = 0; i < T; ++i) y[i * ld + j] = y[i * ld + j] / sigma;
      c[j] *= sigma;
    }
    __syncthreads();
    // token step: std over the channels of (y - y[i][0]), clamped
    for (int i = warp; i < T; i += kGWarps) {
      float* row = y + i * ld;
      const double sh = row[0];
      double s1 = 0.0;
      for (int j = lane; j < D; j += 32) s1 += static_cast<double>(row[j]) - sh;
      const double mean = warp_sum_d(s1) / D;
      double s2 = 0.0;
      for (int j = lane; j < D; j += 32) {
        const double dd = (static_cast<double>(row[j]) - sh) - mean;
        s2 += dd * dd;
      }
      const float rho = fmaxf(static_cast<float>(sqrt(warp_sum_d(s2) / D)), eps);
      __syncwarp();
      for (int j = lane; j < D; j += 32) row[j] = row[j] / rho;
      if (lane == 0) r[i] *= rho;
    }
    __syncthreads();
    // (C, R) -> (C / 2^(e-1), R 2^(e-1)) with max C = m 2^e, m in [0.5, 1)
    float cm = 0.f;
    for (int j = tid; j < D; j += kGThreads) cm = fmaxf(cm, c[j]);
    int e = 0;
    frexpf(block_max(cm, red), &e);
    for (int j = tid; j < D; j += kGThreads) c[j] = ldexpf(c[j], 1 - e);
    for (int i = tid; i < T; i += kGThreads) r[i] = ldexpf(r[i], e - 1);
    __syncthreads();
  }

  // RTN per token (warp per row), codes into the staged pages, s~ = s R and z~ = z R
  for (int i = warp; i < T; i += kGWarps) {
    const float* row = y + i * ld;
    float mn = INFINITY, mx = -INFINITY;
    for (int j = lane; j < D; j += 32) {
      mn = fminf(mn, row[j]);
      mx = fmaxf(mx, row[j]);
    }
    mn = warp_min(mn);
    mx = warp_max(mx);
    const float s = (mx - mn) / static_cast<float>(qmax);
    unsigned char* pg = stage + (i / kPageTokens) * g.page_bytes;
    const int p = i % kPageTokens;
    uint32_t* words = reinterpret_cast<uint32_t*>(pg);
    for (int j = lane; j < D; j += 32) {
      uint32_t code = 0u;
      if (s > 0.f) code = static_cast<uint32_t>(fminf(fmaxf(rintf((row[j] - mn) / s), 0.f), static_cast<float>(qmax)));
      put_code(words, code_bit_d<D>(j, p, bits, is_v), bits, code);
    }
    if (lane == 0)
      *reinterpret_cast<__half2*>(pg + g.meta_off + 4 * p) =
          __halves2half2(__float2half_rn(s * r[i]), __float2half_rn(mn * r[i]));
  }
  // C~ slices: page k of the tile carries channels [k cs, (k + 1) cs)
  for (int j = tid; j < D; j += kGThreads)
    *reinterpret_cast<__half*>(stage + (j / g.cs_channels) * g.page_bytes + g.cslice_off + 2 * (j % g.cs_channels)) =
        __float2half_rn(c[j]);
  __syncthreads();
  const int nh = cfg.num_kv_heads;
  const int per_page = g.page_bytes / 16;
  for (int idx = tid; idx < npages * per_page; idx += kGThreads) {
    const int k = idx / per_page, w = idx % per_page;
    uint4* dst = reinterpret_cast<uint4*>(pool + (static_cast<size_t>(blk[k]) * nh + head) * g.page_bytes);
    dst[w] = reinterpret_cast<const uint4*>(stage + k * g.page_bytes)[w];
  }
  __syncthreads();
}

// Prefill: one CTA per (tile, KV head, K|V) of the descriptor list.
template <int D>
__global__ void __launch_bounds__(kGThreads) gen_quantize_kernel(QuantizeArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int blk[kMaxPages];
  __shared__ int ok;
  const int tile = blockIdx.x, head = blockIdx.y, kv = blockIdx.z;
  const __half* src = static_cast<const __half*>(kv ? a.src_v : a.src_k);
  if (src == nullptr) return;
  const int T = a.cfg.tile_tokens, npages = T / kPageTokens, nh = a.cfg.num_kv_heads;
  const int src_row = a.tile_desc[3 * tile], seq = a.tile_desc[3 * tile + 1], tidx = a.tile_desc[3 * tile + 2];
  if (threadIdx.x == 0) {
    bool good = src_row >= 0 && src_row <= a.num_rows - T && seq >= 0 && seq < a.num_seqs && tidx >= 0 &&
                (tidx + 1) * npages <= a.max_blocks_per_seq;
    for (int k = 0; good && k < npages; ++k) {
      blk[k] = a.block_tables[static_cast<size_t>(seq) * a.max_blocks_per_seq + tidx * npages + k];
      good = blk[k] >= 0 && blk[k] < a.num_blocks;
    }
    if (!good && head == 0 && kv == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
    ok = good;
  }
  __syncthreads();
  if (!ok) return;
  auto row_of = [&](int i) { return src + (static_cast<size_t>(src_row + i) * nh + head) * D; };
  quantize_tile_generic<D>(row_of, T, kv != 0, a.cfg, kv ? a.gv : a.gk, blk,
                           static_cast<uint8_t*>(kv ? a.v_pool : a.k_pool), head, smem);
}

// Append: one CTA per (sequence, KV head, K|V).  Tiles the new tokens
// complete are quantized from the tail rows and the new rows, in order; the
// tokens of the unfinished tile then go to the tail (token q in row q mod T).
template <int D>
__global__ void __launch_bounds__(kGThreads) gen_append_kernel(AppendArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ int blk[kMaxPages];
  __shared__ int ok;
  const int b = blockIdx.x, head = blockIdx.y, kv = blockIdx.z;
  const __half* src = static_cast<const __half*>(kv ? a.new_v : a.new_k);
  __half* tail = static_cast<__half*>(kv ? a.v_tail : a.k_tail);
  if (src == nullptr || tail == nullptr) return;
  const int T = a.cfg.tile_tokens, npages = T / kPageTokens, nh = a.cfg.num_kv_heads;
  const int l0 = a.seq_lens_before[b];
  const int start = a.cu_new[b];
  const int n = a.cu_new[b + 1] - start;
  if (n <= 0 || l0 < 0) return;
  const int end = l0 + n;
  __half* tail_base = tail + (static_cast<size_t>(b) * nh + head) * T * D;
  for (int t = l0 / T; t < end / T; ++t) {
    if (threadIdx.x == 0) {
      bool good = (t + 1) * npages <= a.max_blocks_per_seq;
      for (int k = 0; good && k < npages; ++k) {
        blk[k] = a.block_tables[static_cast<size_t>(b) * a.max_blocks_per_seq + t * npages + k];
        good = blk[k] >= 0 && blk[k] < a.num_blocks;
      }
      if (!good) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
      ok = good;
    }
    __syncthreads();
    if (ok) {
      auto row_of = [&](int i) {
        const int q = t * T + i;
        return q < l0 ? tail_base + static_cast<size_t>(q % T) * D
                      : src + (static_cast<size_t>(start + q - l0) * nh + head) * D;
      };
      quantize_tile_generic<D>(row_of, T, kv != 0, a.cfg, kv ? a.gv : a.gk, blk,
                               static_cast<uint8_t*>(kv ? a.v_pool : a.k_pool), head, smem);
    }
    __syncthreads();
  }
  const int first = max(l0, (end / T) * T);
  const int count = end - first;
  for (int idx = threadIdx.x; idx < count * (D / 8); idx += kGThreads) {
    const int rr = idx / (D / 8), piece = idx % (D / 8);
    const int q = first + rr;
    const uint4 v = *reinterpret_cast<const uint4*>(src + (static_cast<size_t>(start + q - l0) * nh + head) * D +
                                                    8 * piece);
    *reinterpret_cast<uint4*>(tail_base + static_cast<size_t>(q % T) * D + 8 * piece) = v;
  }
}

// ------------------------------------------------------------------ decode
// Split-K decode in the rotated domain, then a merge.  Split kernel: one CTA
// per (sequence, KV head, split) over a run of whole tiles, all g query heads
// together.  Per tile: codes unpacked to shared memory, q'' = q' C~K and
// sigma = sum q'', scores s~ (q'' . code) + z~ sigma (log2 domain), a running
// softmax per head, and acc' += C~V (sum_i p_i s~_i code_i + sum_i p_i z~_i).
// Writes (m, l, acc') per query head.  Merge kernel: one CTA per (sequence,
// KV head): the raw fp16 tail in the original domain, the log-sum-exp merge
// of the splits, the one inverse rotation, fp16 output.
// Partial record: m, l, two pad floats, acc'[D].

template <int D>
constexpr int rec_floats() {
  return 4 + D;
}

// number of splits of the decode on a device with `sms` SMs
int gen_splits(int num_seqs, int num_kv_heads, int num_splits, int sms) {
  if (num_splits > 0) return num_splits;
  const long long pairs = std::max(1LL, static_cast<long long>(num_seqs) * num_kv_heads);
  return static_cast<int>(std::max(1LL, std::min(64LL, (2LL * sms + pairs - 1) / pairs)));
}

// shared memory of the split kernel
struct GenDecSmem {
  size_t qr, qq, acc, sc, ck, cv, mk, mv, hs, kc, vc, total;
};
__host__ __device__ inline GenDecSmem gen_dec_smem(int D, int T) {
  GenDecSmem m;
  const size_t G = kMaxGroup;
  m.qr = 0;                                  // q' [G][D] fp32
  m.qq = m.qr + G * D * 4;                   // q'' [G][D]
  m.acc = m.qq + G * D * 4;                  // acc' [G][D]
  m.sc = m.acc + G * D * 4;                  // scores / p s~V [G][T]
  m.ck = m.sc + G * T * 4;                   // C~K [D]
  m.cv = m.ck + D * 4;                       // C~V [D]
  m.mk = m.cv + D * 4;                       // (s~, z~) of K [T] float2
  m.mv = m.mk + T * 8;                       // (s~, z~) of V [T]
  m.hs = m.mv + T * 8;                       // per head: m, l, alpha, sigma, w [G][8]
  m.kc = m.hs + G * 8 * 4;                   // K codes [T][D + 4] bytes
  m.vc = m.kc + static_cast<size_t>(T) * (D + 4);  // V codes [T][D + 4]
  m.total = m.vc + static_cast<size_t>(T) * (D + 4);
  return m;
}

template <int D>
__global__ void __launch_bounds__(kGThreads) gen_decode_split_kernel(DecodeArgs a, int S) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ const uint8_t* kpg[kMaxPages];
  __shared__ const uint8_t* vpg[kMaxPages];
  __shared__ int ok;
  const int T = a.cfg.tile_tokens, npages = T / kPageTokens;
  const int nh = a.cfg.num_kv_heads, G = a.cfg.group_size;
  const GenDecSmem L = gen_dec_smem(D, T);
  float* qr = reinterpret_cast<float*>(smem + L.qr);
  float* qq = reinterpret_cast<float*>(smem + L.qq);
  float* acc = reinterpret_cast<float*>(smem + L.acc);
  float* sc = reinterpret_cast<float*>(smem + L.sc);
  float* ck = reinterpret_cast<float*>(smem + L.ck);
  float* cv = reinterpret_cast<float*>(smem + L.cv);
  float2* mk = reinterpret_cast<float2*>(smem + L.mk);
  float2* mv = reinterpret_cast<float2*>(smem + L.mv);
  float* hs = reinterpret_cast<float*>(smem + L.hs);  // [G][8]: m, l, alpha, sigma, w
  uint8_t* kc = smem + L.kc;
  uint8_t* vc = smem + L.vc;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = blockIdx.x, split = blockIdx.y;
  const int b = pair / nh, h = pair % nh;
  const int F = max(a.seq_lens[b], 0) / T;
  const int ch = (F + S - 1) / S;
  const int t0 = min(F, split * ch), t1 = min(F, t0 + ch);
  const float qscale = a.softmax_scale * kLog2e * inv_sqrt_d<D>();

  // q' = q D_s H / sqrt(D), times the softmax scale (log2 domain)
  const __half* q = static_cast<const __half*>(a.q) + static_cast<size_t>(pair) * G * D;
  for (int idx = tid; idx < G * D; idx += kGThreads)
    qr[idx] = __half2float(q[idx]) * rotation_sign(a.cfg.rotation_seed, idx % D);
  for (int idx = tid; idx < G * D; idx += kGThreads) acc[idx] = 0.f;
  if (tid < G) {
    hs[8 * tid] = -INFINITY;
    hs[8 * tid + 1] = 0.f;
  }
  __syncthreads();
  fwht_rows<D>(qr, G, D);
  for (int idx = tid; idx < G * D; idx += kGThreads) qr[idx] *= qscale;
  __syncthreads();

  const uint8_t* kpool = static_cast<const uint8_t*>(a.k_pool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.v_pool);
  const PoolGeom gk = a.gk, gv = a.gv;
  for (int tile = t0; tile < t1; ++tile) {
    if (tid == 0) {
      bool good = (tile + 1) * npages <= a.max_blocks_per_seq;
      for (int k = 0; good && k < npages; ++k) {
        const int blk = a.block_tables[static_cast<size_t>(b) * a.max_blocks_per_seq + tile * npages + k];
        good = blk >= 0 && blk < a.num_blocks;
        if (good) {
          kpg[k] = kpool + (static_cast<size_t>(blk) * nh + h) * gk.page_bytes;
          vpg[k] = vpool + (static_cast<size_t>(blk) * nh + h) * gv.page_bytes;
        }
      }
      if (!good) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
      ok = good;
    }
    __syncthreads();
    const bool tile_ok = ok;
    __syncthreads();  // every thread has read ok before thread 0 writes the next tile's
    if (!tile_ok) continue;  // tile skipped (reported)
    // codes, metadata and C~ of the tile
    for (int idx = tid; idx < T * D; idx += kGThreads) {
      const int i = idx / D, j = idx % D, k = i / kPageTokens, p = i % kPageTokens;
      kc[i * (D + 4) + j] = static_cast<uint8_t>(read_code(kpg[k], code_bit_d<D>(j, p, gk.bits, false), gk.bits));
      vc[i * (D + 4) + j] = static_cast<uint8_t>(read_code(vpg[k], code_bit_d<D>(j, p, gv.bits, true), gv.bits));
    }
    for (int i = tid; i < T; i += kGThreads) {
      const int k = i / kPageTokens, p = i % kPageTokens;
      mk[i] = __half22float2(*reinterpret_cast<const __half2*>(kpg[k] + gk.meta_off + 4 * p));
      mv[i] = __half22float2(*reinterpret_cast<const __half2*>(vpg[k] + gv.meta_off + 4 * p));
    }
    for (int j = tid; j < D; j += kGThreads) {
      ck[j] = __half2float(*reinterpret_cast<const __half*>(kpg[j / gk.cs_channels] + gk.cslice_off +
                                                            2 * (j % gk.cs_channels)));
      cv[j] = __half2float(*reinterpret_cast<const __half*>(vpg[j / gv.cs_channels] + gv.cslice_off +
                                                            2 * (j % gv.cs_channels)));
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kGThreads) qq[idx] = qr[idx] * ck[idx % D];
    __syncthreads();
    for (int hh = warp; hh < G; hh += kGWarps) {  // sigma = sum_j q''_j
      float sg = 0.f;
      for (int j = lane; j < D; j += 32) sg += qq[hh * D + j];
      sg = warp_sum(sg);
      if (lane == 0) hs[8 * hh + 3] = sg;
    }
    __syncthreads();
    for (int idx = tid; idx < G * T; idx += kGThreads) {  // scores
      const int hh = idx / T, i = idx % T;
      const float* qh = qq + hh * D;
      const uint8_t* ci = kc + i * (D + 4);
      float dot = 0.f;
      for (int j = 0; j < D; j += 4) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(ci + j);
        dot += qh[j] * static_cast<float>(w & 0xffu) + qh[j + 1] * static_cast<float>((w >> 8) & 0xffu) +
               qh[j + 2] * static_cast<float>((w >> 16) & 0xffu) + qh[j + 3] * static_cast<float>(w >> 24);
      }
      sc[hh * T + i] = mk[i].x * dot + mk[i].y * hs[8 * hh + 3];
    }
    __syncthreads();
    for (int hh = warp; hh < G; hh += kGWarps) {  // running softmax; P' = p s~V, w = sum p z~V
      float tm = -INFINITY;
      for (int i = lane; i < T; i += 32) tm = fmaxf(tm, sc[hh * T + i]);
      tm = warp_max(tm);
      const float m_old = hs[8 * hh], m_new = fmaxf(m_old, tm);
      const float alpha = exp2f(m_old - m_new);
      float ls = 0.f, wz = 0.f;
      for (int i = lane; i < T; i += 32) {
        const float pv = exp2f(sc[hh * T + i] - m_new);
        ls += pv;
        wz += pv * mv[i].y;
        sc[hh * T + i] = pv * mv[i].x;
      }
      ls = warp_sum(ls);
      wz = warp_sum(wz);
      if (lane == 0) {
        hs[8 * hh] = m_new;
        hs[8 * hh + 1] = hs[8 * hh + 1] * alpha + ls;
        hs[8 * hh + 2] = alpha;
        hs[8 * hh + 4] = wz;
      }
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += kGThreads) {  // P V
      const int hh = idx / D, j = idx % D;
      const float* ph = sc + hh * T;
      float u = 0.f;
      for (int i = 0; i < T; ++i) u += ph[i] * static_cast<float>(vc[i * (D + 4) + j]);
      acc[idx] = hs[8 * hh + 2] * acc[idx] + cv[j] * (u + hs[8 * hh + 4]);
    }
    __syncthreads();
  }
  float* rec = static_cast<float*>(a.workspace) + (static_cast<size_t>(pair) * S + split) * G * rec_floats<D>();
  for (int idx = tid; idx < G * D; idx += kGThreads) rec[(idx / D) * rec_floats<D>() + 4 + idx % D] = acc[idx];
  if (tid < G) {
    rec[tid * rec_floats<D>()] = hs[8 * tid];
    rec[tid * rec_floats<D>() + 1] = hs[8 * tid + 1];
  }
}

// shared memory of the merge kernel: acc [G][D], acc of the tail [G][D], the
// raw query [G][D], tail scores [G][T], per head scalars [G][8]
__host__ __device__ inline size_t gen_merge_smem(int D, int T) {
  return (3 * static_cast<size_t>(kMaxGroup) * D + static_cast<size_t>(kMaxGroup) * T + kMaxGroup * 8) * 4;
}

template <int D>
__global__ void __launch_bounds__(kGThreads) gen_decode_merge_kernel(DecodeArgs a, int S) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int T = a.cfg.tile_tokens, nh = a.cfg.num_kv_heads, G = a.cfg.group_size;
  float* acc = reinterpret_cast<float*>(smem);
  float* at = acc + kMaxGroup * D;
  float* qs = at + kMaxGroup * D;
  float* ts = qs + kMaxGroup * D;
  float* hs = ts + kMaxGroup * T;  // [G][8]: tail m, tail l, merged m, total l, tail weight
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pair = blockIdx.x, b = pair / nh;
  const int L = max(a.seq_lens[b], 0), tau = L % T;
  const float qscale = a.softmax_scale * kLog2e;
  const __half* kt = static_cast<const __half*>(a.k_tail) + static_cast<size_t>(pair) * T * D;
  const __half* vt = static_cast<const __half*>(a.v_tail) + static_cast<size_t>(pair) * T * D;
  const __half* q = static_cast<const __half*>(a.q) + static_cast<size_t>(pair) * G * D;

  // raw tail, original domain: scores q . k (scaled, log2), softmax over the tail, P V
  for (int idx = tid; idx < G * D; idx += kGThreads) qs[idx] = __half2float(q[idx]) * qscale;
  __syncthreads();
  for (int idx = tid; idx < G * tau; idx += kGThreads) {
    const int hh = idx / tau, i = idx % tau;
    const __half* kr = kt + static_cast<size_t>(i) * D;
    float dot = 0.f;
    for (int j = 0; j < D; ++j) dot += qs[hh * D + j] * __half2float(kr[j]);
    ts[hh * T + i] = dot;
  }
  __syncthreads();
  for (int hh = warp; hh < G; hh += kGWarps) {
    float tm = -INFINITY;
    for (int i = lane; i < tau; i += 32) tm = fmaxf(tm, ts[hh * T + i]);
    tm = warp_max(tm);
    float ls = 0.f;
    for (int i = lane; i < tau; i += 32) {
      const float pv = exp2f(ts[hh * T + i] - tm);
      ts[hh * T + i] = pv;
      ls += pv;
    }
    ls = warp_sum(ls);
    if (lane == 0) {
      hs[8 * hh] = tm;
      hs[8 * hh + 1] = ls;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kGThreads) {
    const int hh = idx / D, j = idx % D;
    float u = 0.f;
    for (int i = 0; i < tau; ++i) u += ts[hh * T + i] * __half2float(vt[static_cast<size_t>(i) * D + j]);
    at[idx] = u;
  }
  // merged maximum, the weights of the splits and the tail, total l
  const float* recs = static_cast<const float*>(a.workspace) + static_cast<size_t>(pair) * S * G * rec_floats<D>();
  for (int hh = warp; hh < G; hh += kGWarps) {
    float mm = hs[8 * hh + 1] > 0.f ? hs[8 * hh] : -INFINITY;
    for (int s2 = lane; s2 < S; s2 += 32) {
      const float* r = recs + (static_cast<size_t>(s2) * G + hh) * rec_floats<D>();
      if (r[1] > 0.f) mm = fmaxf(mm, r[0]);
    }
    mm = warp_max(mm);
    float ls = 0.f;
    for (int s2 = lane; s2 < S; s2 += 32) {
      const float* r = recs + (static_cast<size_t>(s2) * G + hh) * rec_floats<D>();
      if (r[1] > 0.f) ls += exp2f(r[0] - mm) * r[1];
    }
    ls = warp_sum(ls);
    if (lane == 0) {
      const float et = hs[8 * hh + 1] > 0.f ? exp2f(hs[8 * hh] - mm) : 0.f;
      hs[8 * hh + 2] = mm;
      hs[8 * hh + 3] = ls + et * hs[8 * hh + 1];
      hs[8 * hh + 4] = et;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < G * D; idx += kGThreads) {
    const int hh = idx / D, j = idx % D;
    const float mm = hs[8 * hh + 2];
    float u = 0.f;
    for (int s2 = 0; s2 < S; ++s2) {
      const float* r = recs + (static_cast<size_t>(s2) * G + hh) * rec_floats<D>();
      if (r[1] > 0.f) u += exp2f(r[0] - mm) * r[4 + j];
    }
    acc[idx] = u;
  }
  __syncthreads();
  fwht_rows<D>(acc, G, D);  // the one inverse rotation: acc' H D_s / sqrt(D)
  __half* out = static_cast<__half*>(a.out) + static_cast<size_t>(pair) * G * D;
  for (int idx = tid; idx < G * D; idx += kGThreads) {
    const int hh = idx / D, j = idx % D;
    const float ltot = hs[8 * hh + 3];
    const float inv_l = ltot > 0.f ? 1.f / ltot : 0.f;
    const float o = acc[idx] * inv_sqrt_d<D>() * rotation_sign(a.cfg.rotation_seed, j) + hs[8 * hh + 4] * at[idx];
    out[idx] = __float2half_rn(o * inv_l);
  }
}

// ------------------------------------------------------------------ serving step
// The step's token of every sequence into its tail, then the lengths advanced
// by one (one CTA per sequence: every thread reads the length before thread 0
// rewrites it).  A token that would complete a tile is refused (reported and
// not written), as in the one-launch step at d = 128; the length still
// advances.  The decode of the step follows as its own launches.
template <int D>
__global__ void __launch_bounds__(kGThreads) gen_step_append_kernel(DecodeArgs a) {
  const int b = blockIdx.x, T = a.cfg.tile_tokens, nh = a.cfg.num_kv_heads;
  const int L = max(a.seq_lens[b], 0) + 1;  // length with the step's token
  __syncthreads();
  if (L % T == 0) {
    if (threadIdx.x == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
  } else {
    const int row = (L - 1) % T;
    for (int idx = threadIdx.x; idx < nh * (D / 8); idx += kGThreads) {
      const int h = idx / (D / 8), piece = idx % (D / 8);
      const size_t bh = static_cast<size_t>(b) * nh + h;
      const size_t src = bh * D + 8 * piece, dst = (bh * T + row) * D + 8 * piece;
      *reinterpret_cast<uint4*>(static_cast<__half*>(const_cast<void*>(a.k_tail)) + dst) =
          *reinterpret_cast<const uint4*>(static_cast<const __half*>(a.new_k) + src);
      *reinterpret_cast<uint4*>(static_cast<__half*>(const_cast<void*>(a.v_tail)) + dst) =
          *reinterpret_cast<const uint4*>(static_cast<const __half*>(a.new_v) + src);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) a.seq_lens_rw[b] = L;
}

// ------------------------------------------------------------------ prefill
// Chunked prefill attention (aitrends.kr article 74976, "TL;DR": every phase
// of attention reads the compressed pages directly): chunk token i of a
// sequence attends to its cached context (full tiles from the pages, in the
// rotated domain, as the decode split kernel reads them; then the raw fp16
// tail) and, causally, to the chunk's own raw rows 0..i.  One CTA per
// (sequence, KV head, run of chunk tokens); its query rows are those tokens
// x the g query heads of the KV head, token-major (row r: token r / g, head
// r % g).  Two running softmax states per row, one per domain: the context
// tiles in the rotated domain, the tail and chunk rows in the original one;
// the rotated accumulator goes back through one inverse rotation, then the
// two states are merged by their log-sum-exp weights.

constexpr int kPfRawBlk = 16;  // raw keys per block of the original-domain phase

template <int D>
constexpr int gen_pf_rows() {
  return D == 64 ? 32 : 16;  // query rows per CTA
}

struct GenPfSmem {
  size_t qr, qq, acc, acc2, sc, ck, cv, mk, mv, hs, kc, vc, total;
};
__host__ __device__ inline GenPfSmem gen_pf_smem(int D, int T, int R) {
  GenPfSmem m;
  const size_t rd = static_cast<size_t>(R) * D * 4;
  m.qr = 0;                                  // q' (then the scaled raw q) [R][D] fp32
  m.qq = m.qr + rd;                          // q'' [R][D]
  m.acc = m.qq + rd;                         // acc' (rotated domain) [R][D]
  m.acc2 = m.acc + rd;                       // acc (original domain) [R][D]
  m.sc = m.acc2 + rd;                        // scores / p [R][T]
  m.ck = m.sc + static_cast<size_t>(R) * T * 4;
  m.cv = m.ck + D * 4;
  m.mk = m.cv + D * 4;                       // (s~, z~) of K [T] float2
  m.mv = m.mk + T * 8;
  m.hs = m.mv + T * 8;                       // per row [R][8]: m, l, alpha, sigma, w, m2, l2, -
  m.kc = m.hs + static_cast<size_t>(R) * 8 * 4;  // K codes [T][D + 4] bytes, or raw K rows [16][D] fp16
  m.vc = m.kc + static_cast<size_t>(T) * (D + 4);
  m.total = m.vc + static_cast<size_t>(T) * (D + 4);
  return m;
}

// CTAs of a prefill launch: (sequences x KV heads) x runs of chunk tokens
long long gen_pf_ctas(const kvq_config& cfg, int num_seqs, int max_chunk) {
  const int R = cfg.head_dim == 64 ? gen_pf_rows<64>() : gen_pf_rows<256>();
  const long long toks = std::max(1, R / cfg.group_size);
  return static_cast<long long>(num_seqs) * cfg.num_kv_heads * ((max_chunk + toks - 1) / toks);
}

// Running softmax over one block of `n` score columns per row (log2 domain):
// new maximum, alpha = 2^(m_old - m_new), p = 2^(s - m_new) written back, row
// sums added into l; masked columns hold -inf and give p = 0.
__device__ __forceinline__ void pf_softmax_rows(float* sc, int ld, int n, int rows, float* hs, int im, int il) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int r = warp; r < rows; r += kGWarps) {
    float tm = -INFINITY;
    for (int i = lane; i < n; i += 32) tm = fmaxf(tm, sc[r * ld + i]);
    tm = warp_max(tm);
    const float m_old = hs[8 * r + im], m_new = fmaxf(m_old, tm);
    const float alpha = m_new == -INFINITY ? 1.f : exp2f(m_old - m_new);
    float ls = 0.f;
    for (int i = lane; i < n; i += 32) {
      const float s = sc[r * ld + i];
      const float pv = s == -INFINITY ? 0.f : exp2f(s - m_new);
      sc[r * ld + i] = pv;
      ls += pv;
    }
    ls = warp_sum(ls);
    if (lane == 0) {
      hs[8 * r + im] = m_new;
      hs[8 * r + il] = hs[8 * r + il] * alpha + ls;
      hs[8 * r + 2] = alpha;
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kGThreads) gen_prefill_kernel(PrefillArgs a, PoolGeom gk, PoolGeom gv) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ const uint8_t* kpg[kMaxPages];
  __shared__ const uint8_t* vpg[kMaxPages];
  __shared__ int ok;
  constexpr int R = gen_pf_rows<D>();
  const int T = a.cfg.tile_tokens, npages = T / kPageTokens;
  const int nh = a.cfg.num_kv_heads, G = a.cfg.group_size, Hq = nh * G;
  const int toks = max(1, R / G), rows = toks * G;  // chunk tokens and query rows of this CTA
  const GenPfSmem L = gen_pf_smem(D, T, R);
  float* qr = reinterpret_cast<float*>(smem + L.qr);
  float* qq = reinterpret_cast<float*>(smem + L.qq);
  float* acc = reinterpret_cast<float*>(smem + L.acc);
  float* acc2 = reinterpret_cast<float*>(smem + L.acc2);
  float* sc = reinterpret_cast<float*>(smem + L.sc);
  float* ck = reinterpret_cast<float*>(smem + L.ck);
  float* cv = reinterpret_cast<float*>(smem + L.cv);
  float2* mk = reinterpret_cast<float2*>(smem + L.mk);
  float2* mv = reinterpret_cast<float2*>(smem + L.mv);
  float* hs = reinterpret_cast<float*>(smem + L.hs);
  uint8_t* kc = smem + L.kc;
  uint8_t* vc = smem + L.vc;
  const int tid = threadIdx.x;
  const int runs = (a.max_chunk + toks - 1) / toks;
  const int pair = static_cast<int>(blockIdx.x / runs), run = static_cast<int>(blockIdx.x % runs);
  const int b = pair / nh, h = pair % nh;
  const int c0 = a.cu_chunk[b];
  const int n = a.cu_chunk[b + 1] - c0;
  if ((n < 0 || n > a.max_chunk) && tid == 0 && run == 0 && h == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
  const int nc = max(0, min(n, a.max_chunk));  // chunk tokens served
  const int i0 = run * toks;
  if (i0 >= nc) return;
  const int nt = min(toks, nc - i0);  // live tokens of this CTA; rows >= nt * G are idle
  const int Lc = max(a.ctx_lens[b], 0), F = Lc / T, tau = Lc % T;
  const float qscale = a.softmax_scale * kLog2e;
  const __half* q = static_cast<const __half*>(a.q);

  // q' = q D_s H / sqrt(D) times the softmax scale (log2 domain); idle rows 0
  for (int idx = tid; idx < rows * D; idx += kGThreads) {
    const int r = idx / D, j = idx % D, ti = r / G;
    const float v = ti < nt ? __half2float(q[(static_cast<size_t>(c0 + i0 + ti) * Hq + h * G + r % G) * D + j]) : 0.f;
    qr[idx] = v * rotation_sign(a.cfg.rotation_seed, j);
    acc[idx] = 0.f;
    acc2[idx] = 0.f;
  }
  for (int r = tid; r < rows; r += kGThreads) {
    hs[8 * r] = -INFINITY;
    hs[8 * r + 1] = 0.f;
    hs[8 * r + 5] = -INFINITY;
    hs[8 * r + 6] = 0.f;
  }
  __syncthreads();
  fwht_rows<D>(qr, rows, D);
  for (int idx = tid; idx < rows * D; idx += kGThreads) qr[idx] *= qscale * inv_sqrt_d<D>();
  __syncthreads();

  // ---- context tiles, rotated domain
  const uint8_t* kpool = static_cast<const uint8_t*>(a.k_pool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.v_pool);
  for (int tile = 0; tile < F; ++tile) {
    if (tid == 0) {
      bool good = (tile + 1) * npages <= a.max_blocks_per_seq;
      for (int k = 0; good && k < npages; ++k) {
        const int blk = a.block_tables[static_cast<size_t>(b) * a.max_blocks_per_seq + tile * npages + k];
        good = blk >= 0 && blk < a.num_blocks;
        if (good) {
          kpg[k] = kpool + (static_cast<size_t>(blk) * nh + h) * gk.page_bytes;
          vpg[k] = vpool + (static_cast<size_t>(blk) * nh + h) * gv.page_bytes;
        }
      }
      if (!good) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
      ok = good;
    }
    __syncthreads();
    const bool tile_ok = ok;
    __syncthreads();  // every thread has read ok before thread 0 writes the next tile's
    if (!tile_ok) continue;  // tile skipped (reported)
    for (int idx = tid; idx < T * D; idx += kGThreads) {
      const int i = idx / D, j = idx % D, k = i / kPageTokens, p = i % kPageTokens;
      kc[i * (D + 4) + j] = static_cast<uint8_t>(read_code(kpg[k], code_bit_d<D>(j, p, gk.bits, false), gk.bits));
      vc[i * (D + 4) + j] = static_cast<uint8_t>(read_code(vpg[k], code_bit_d<D>(j, p, gv.bits, true), gv.bits));
    }
    for (int i = tid; i < T; i += kGThreads) {
      const int k = i / kPageTokens, p = i % kPageTokens;
      mk[i] = __half22float2(*reinterpret_cast<const __half2*>(kpg[k] + gk.meta_off + 4 * p));
      mv[i] = __half22float2(*reinterpret_cast<const __half2*>(vpg[k] + gv.meta_off + 4 * p));
    }
    for (int j = tid; j < D; j += kGThreads) {
      ck[j] = __half2float(*reinterpret_cast<const __half*>(kpg[j / gk.cs_channels] + gk.cslice_off +
                                                            2 * (j % gk.cs_channels)));
      cv[j] = __half2float(*reinterpret_cast<const __half*>(vpg[j / gv.cs_channels] + gv.cslice_off +
                                                            2 * (j % gv.cs_channels)));
    }
    __syncthreads();
    for (int idx = tid; idx < rows * D; idx += kGThreads) qq[idx] = qr[idx] * ck[idx % D];
    __syncthreads();
    for (int r = threadIdx.x >> 5; r < rows; r += kGWarps) {  // sigma = sum_j q''_j
      float sg = 0.f;
      for (int j = threadIdx.x & 31; j < D; j += 32) sg += qq[r * D + j];
      sg = warp_sum(sg);
      if ((threadIdx.x & 31) == 0) hs[8 * r + 3] = sg;
    }
    __syncthreads();
    for (int idx = tid; idx < rows * T; idx += kGThreads) {  // scores s~ (q'' . code) + z~ sigma
      const int r = idx / T, i = idx % T;
      const float* qh = qq + r * D;
      const uint8_t* ci = kc + i * (D + 4);
      float dot = 0.f;
      for (int j = 0; j < D; j += 4) {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(ci + j);
        dot += qh[j] * static_cast<float>(w & 0xffu) + qh[j + 1] * static_cast<float>((w >> 8) & 0xffu) +
               qh[j + 2] * static_cast<float>((w >> 16) & 0xffu) + qh[j + 3] * static_cast<float>(w >> 24);
      }
      sc[r * T + i] = mk[i].x * dot + mk[i].y * hs[8 * r + 3];
    }
    __syncthreads();
    pf_softmax_rows(sc, T, T, rows, hs, 0, 1);
    __syncthreads();
    for (int r = threadIdx.x >> 5; r < rows; r += kGWarps) {  // P' = p s~V in place, w = sum p z~V
      float wz = 0.f;
      for (int i = threadIdx.x & 31; i < T; i += 32) {
        const float pv = sc[r * T + i];
        wz += pv * mv[i].y;
        sc[r * T + i] = pv * mv[i].x;
      }
      wz = warp_sum(wz);
      if ((threadIdx.x & 31) == 0) hs[8 * r + 4] = wz;
    }
    __syncthreads();
    for (int idx = tid; idx < rows * D; idx += kGThreads) {  // acc' = alpha acc' + C~V (P' code + w)
      const int r = idx / D, j = idx % D;
      const float* ph = sc + r * T;
      float u = 0.f;
      for (int i = 0; i < T; ++i) u += ph[i] * static_cast<float>(vc[i * (D + 4) + j]);
      acc[idx] = hs[8 * r + 2] * acc[idx] + cv[j] * (u + hs[8 * r + 4]);
    }
    __syncthreads();
  }

  // ---- raw keys, original domain: the tail (positions F T .. Lc - 1, tail
  // rows 0 .. tau - 1), then chunk rows 0 .. i0 + nt - 1, causal per row
  for (int idx = tid; idx < rows * D; idx += kGThreads) {
    const int r = idx / D, j = idx % D, ti = r / G;
    qr[idx] = ti < nt ? __half2float(q[(static_cast<size_t>(c0 + i0 + ti) * Hq + h * G + r % G) * D + j]) * qscale
                      : 0.f;
  }
  const __half* kt = static_cast<const __half*>(a.k_tail) + static_cast<size_t>(pair) * T * D;
  const __half* vt = static_cast<const __half*>(a.v_tail) + static_cast<size_t>(pair) * T * D;
  const __half* kn = static_cast<const __half*>(a.k_new);
  const __half* vn = static_cast<const __half*>(a.v_new);
  __half* kr = reinterpret_cast<__half*>(kc);  // [16][D]
  __half* vr = reinterpret_cast<__half*>(vc);
  const int nkeys = tau + i0 + nt;
  for (int u0 = 0; u0 < nkeys; u0 += kPfRawBlk) {
    const int nb = min(kPfRawBlk, nkeys - u0);
    __syncthreads();  // the previous block's rows are no longer read
    for (int idx = tid; idx < nb * (D / 8); idx += kGThreads) {
      const int i = idx / (D / 8), piece = idx % (D / 8), u = u0 + i;
      const size_t src = u < tau ? static_cast<size_t>(u) * D
                                 : (static_cast<size_t>(c0 + u - tau) * nh + h) * D;
      const __half* ks = u < tau ? kt : kn;
      const __half* vs = u < tau ? vt : vn;
      *reinterpret_cast<uint4*>(kr + i * D + 8 * piece) = *reinterpret_cast<const uint4*>(ks + src + 8 * piece);
      *reinterpret_cast<uint4*>(vr + i * D + 8 * piece) = *reinterpret_cast<const uint4*>(vs + src + 8 * piece);
    }
    __syncthreads();
    for (int idx = tid; idx < rows * kPfRawBlk; idx += kGThreads) {
      const int r = idx / kPfRawBlk, i = idx % kPfRawBlk, u = u0 + i;
      const int ti = i0 + r / G;  // chunk index of the row's token
      float s = -INFINITY;
      if (i < nb && (u < tau || u - tau <= ti)) {
        s = 0.f;
        for (int j = 0; j < D; ++j) s += qr[r * D + j] * __half2float(kr[i * D + j]);
      }
      sc[r * T + i] = s;
    }
    __syncthreads();
    pf_softmax_rows(sc, T, kPfRawBlk, rows, hs, 5, 6);
    __syncthreads();
    for (int idx = tid; idx < rows * D; idx += kGThreads) {
      const int r = idx / D, j = idx % D;
      float u = 0.f;
      for (int i = 0; i < nb; ++i) u += sc[r * T + i] * __half2float(vr[i * D + j]);
      acc2[idx] = hs[8 * r + 2] * acc2[idx] + u;
    }
  }
  __syncthreads();

  // ---- the one inverse rotation of the context part, the log-sum-exp merge, fp16 out
  fwht_rows<D>(acc, rows, D);
  __half* out = static_cast<__half*>(a.out);
  for (int idx = tid; idx < nt * G * D; idx += kGThreads) {
    const int r = idx / D, j = idx % D;
    const float m1 = hs[8 * r], l1 = hs[8 * r + 1], m2 = hs[8 * r + 5], l2 = hs[8 * r + 6];
    const float mm = fmaxf(m1, m2);
    const float e1 = l1 > 0.f ? exp2f(m1 - mm) : 0.f, e2 = l2 > 0.f ? exp2f(m2 - mm) : 0.f;
    const float ltot = e1 * l1 + e2 * l2;
    const float o = e1 * acc[idx] * inv_sqrt_d<D>() * rotation_sign(a.cfg.rotation_seed, j) + e2 * acc2[idx];
    out[(static_cast<size_t>(c0 + i0 + r / G) * Hq + h * G + r % G) * D + j] =
        __float2half_rn(ltot > 0.f ? o / ltot : 0.f);
  }
}

// ------------------------------------------------------------------ read-back
// Codes, metadata, C~ and the dequantized tile in both domains, for one
// (tile, KV head) per CTA.
template <int D>
__global__ void __launch_bounds__(kGThreads) gen_unpack_kernel(UnpackArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ const uint8_t* pages[kMaxPages];
  __shared__ int ok;
  const int T = a.cfg.tile_tokens, npages = T / kPageTokens, nh = a.cfg.num_kv_heads;
  const int tile = blockIdx.x, head = blockIdx.y, tid = threadIdx.x;
  const PoolGeom g = a.g;
  const bool is_v = a.is_v != 0;
  const int seq = a.tile_desc[2 * tile], tidx = a.tile_desc[2 * tile + 1];
  if (tid == 0) {
    bool good = seq >= 0 && seq < a.num_seqs && tidx >= 0 && (tidx + 1) * npages <= a.max_blocks_per_seq;
    for (int k = 0; good && k < npages; ++k) {
      const int blk = a.block_tables[static_cast<size_t>(seq) * a.max_blocks_per_seq + tidx * npages + k];
      good = blk >= 0 && blk < a.num_blocks;
      if (good) pages[k] = static_cast<const uint8_t*>(a.pool) + (static_cast<size_t>(blk) * nh + head) * g.page_bytes;
    }
    if (!good) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
    ok = good;
  }
  __syncthreads();
  if (!ok) return;
  const size_t th = static_cast<size_t>(tile) * nh + head;
  float* y = reinterpret_cast<float*>(smem);  // [T][D]
  for (int idx = tid; idx < T * D; idx += kGThreads) {
    const int i = idx / D, j = idx % D, k = i / kPageTokens, p = i % kPageTokens;
    const int code = read_code(pages[k], code_bit_d<D>(j, p, g.bits, is_v), g.bits);
    const float2 md = __half22float2(*reinterpret_cast<const __half2*>(pages[k] + g.meta_off + 4 * p));
    const __half cj = *reinterpret_cast<const __half*>(pages[j / g.cs_channels] + g.cslice_off +
                                                      2 * (j % g.cs_channels));
    if (a.codes) a.codes[th * T * D + idx] = static_cast<uint8_t>(code);
    if (a.meta && j == 0) static_cast<__half2*>(a.meta)[th * T + i] = __floats2half2_rn(md.x, md.y);
    if (a.cvec && i == 0) static_cast<__half*>(a.cvec)[th * D + j] = cj;
    const float v = (static_cast<float>(code) * md.x + md.y) * __half2float(cj);
    if (a.out_rot) a.out_rot[th * T * D + idx] = v;
    y[idx] = v;
  }
  __syncthreads();
  if (a.out_orig) {
    fwht_rows<D>(y, T, D);
    for (int idx = tid; idx < T * D; idx += kGThreads)
      a.out_orig[th * T * D + idx] = y[idx] * inv_sqrt_d<D>() * rotation_sign(a.cfg.rotation_seed, idx % D);
  }
}

template <class K>
cudaError_t allow_smem(K kern, size_t bytes) {
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes));
}

template <int D>
cudaError_t launch_generic_quantize_d(const QuantizeArgs& a, cudaStream_t s) {
  const size_t smem = gq_smem_bytes(D, a.cfg.tile_tokens, std::max(a.gk.page_bytes, a.gv.page_bytes));
  cudaError_t e = allow_smem(gen_quantize_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  gen_quantize_kernel<D><<<dim3(a.num_tiles, a.cfg.num_kv_heads, 2), kGThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_generic_append_d(const AppendArgs& a, cudaStream_t s) {
  const size_t smem = gq_smem_bytes(D, a.cfg.tile_tokens, std::max(a.gk.page_bytes, a.gv.page_bytes));
  cudaError_t e = allow_smem(gen_append_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  gen_append_kernel<D><<<dim3(a.num_seqs, a.cfg.num_kv_heads, 2), kGThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_generic_decode_d(const DecodeArgs& a, cudaStream_t s, int S) {
  const size_t smem1 = gen_dec_smem(D, a.cfg.tile_tokens).total;
  cudaError_t e = allow_smem(gen_decode_split_kernel<D>, smem1);
  if (e != cudaSuccess) return e;
  const size_t smem2 = gen_merge_smem(D, a.cfg.tile_tokens);
  e = allow_smem(gen_decode_merge_kernel<D>, smem2);
  if (e != cudaSuccess) return e;
  const unsigned pairs = static_cast<unsigned>(a.num_seqs) * a.cfg.num_kv_heads;
  gen_decode_split_kernel<D><<<dim3(pairs, S), kGThreads, smem1, s>>>(a, S);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  gen_decode_merge_kernel<D><<<pairs, kGThreads, smem2, s>>>(a, S);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_generic_prefill_d(const PrefillArgs& a, cudaStream_t s) {
  const size_t smem = gen_pf_smem(D, a.cfg.tile_tokens, gen_pf_rows<D>()).total;
  cudaError_t e = allow_smem(gen_prefill_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  const long long ctas = gen_pf_ctas(a.cfg, a.num_seqs, a.max_chunk);
  gen_prefill_kernel<D><<<static_cast<unsigned>(ctas), kGThreads, smem, s>>>(a, pool_geom(a.cfg, false),
                                                                             pool_geom(a.cfg, true));
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_generic_unpack_d(const UnpackArgs& a, cudaStream_t s) {
  const size_t smem = static_cast<size_t>(a.cfg.tile_tokens) * D * 4;
  cudaError_t e = allow_smem(gen_unpack_kernel<D>, smem);
  if (e != cudaSuccess) return e;
  gen_unpack_kernel<D><<<dim3(a.num_tiles, a.cfg.num_kv_heads), kGThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_generic_quantize(const QuantizeArgs& a, cudaStream_t s) {
  if (a.num_tiles == 0) return cudaSuccess;
  return a.cfg.head_dim == 64 ? launch_generic_quantize_d<64>(a, s) : launch_generic_quantize_d<256>(a, s);
}

cudaError_t launch_generic_append(const AppendArgs& a, cudaStream_t s) {
  if (a.num_seqs == 0) return cudaSuccess;
  return a.cfg.head_dim == 64 ? launch_generic_append_d<64>(a, s) : launch_generic_append_d<256>(a, s);
}

size_t generic_decode_workspace_bytes(const kvq_config& cfg, int num_seqs, int num_splits, int num_sms) {
  const size_t S = static_cast<size_t>(gen_splits(num_seqs, cfg.num_kv_heads, num_splits, num_sms));
  return static_cast<size_t>(num_seqs) * cfg.num_kv_heads * S * cfg.group_size * (4 + cfg.head_dim) * sizeof(float);
}

cudaError_t launch_generic_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.num_seqs == 0) return cudaSuccess;
  int sms = 148;
  if (a.num_splits_fixed == 0) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
  }
  const int S = gen_splits(a.num_seqs, a.cfg.num_kv_heads, a.num_splits_fixed, sms);
  return a.cfg.head_dim == 64 ? launch_generic_decode_d<64>(a, s, S) : launch_generic_decode_d<256>(a, s, S);
}

long long generic_prefill_ctas(const kvq_config& cfg, int num_seqs, int max_chunk) {
  return gen_pf_ctas(cfg, num_seqs, max_chunk);
}

cudaError_t launch_generic_step(const DecodeArgs& a, cudaStream_t s) {
  if (a.num_seqs == 0) return cudaSuccess;
  if (a.cfg.head_dim == 64)
    gen_step_append_kernel<64><<<a.num_seqs, kGThreads, 0, s>>>(a);
  else
    gen_step_append_kernel<256><<<a.num_seqs, kGThreads, 0, s>>>(a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_generic_decode(a, s);
}

cudaError_t launch_generic_prefill(const PrefillArgs& a, cudaStream_t s) {
  if (a.num_seqs == 0 || a.max_chunk == 0) return cudaSuccess;
  return a.cfg.head_dim == 64 ? launch_generic_prefill_d<64>(a, s) : launch_generic_prefill_d<256>(a, s);
}

cudaError_t launch_generic_unpack(const UnpackArgs& a, cudaStream_t s) {
  if (a.num_tiles == 0) return cudaSuccess;
  return a.cfg.head_dim == 64 ? launch_generic_unpack_d<64>(a, s) : launch_generic_unpack_d<256>(a, s);
}

}  // namespace kvq
