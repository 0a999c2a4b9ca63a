// Write path on the 5th-generation tensor cores: tile quantization (prefill)
// and token append with tile completion.
//
// Method: axbrief.com "Huawei's KVarN boosts vLLM KV-cache capacity by 5x
// without accuracy loss", section "What differs from existing methods":
// per fixed-size token tile, Hadamard rotation along the channels, then
// Sinkhorn-like alternating variance normalization, then asymmetric RTN.
//
// A persistent CTA of 8 math warps and 1 producer warp works on a group of
// 128 token rows = 128/T tiles of one (KV head, K|V) at a time; the producer
// warp loads and rotates the next group while the math warps finish the
// current one:
//   load    TMA (cp.async.bulk.tensor, 128-byte swizzle) brings the fp16
//           rows into shared memory; the next group's load is issued as soon
//           as the current group's MMAs have read the buffer
//   rotate  two tcgen05.mma (kind::f16, fp32 accumulate in TMEM) against the
//           +-1 Sylvester matrix: D1 = X H (TMEM lane = token, column =
//           channel) and D2 = H X^T (lane = channel, column = token).  The
//           products are exact and the sums of 128 fp16 values are done in the
//           tensor core's fp32 accumulator.
//   normalize  per iteration, channel statistics stream D2 rows (one channel
//           per thread) and token statistics stream D1 rows (one token per
//           thread) out of TMEM with packed f32x2 arithmetic; the tile itself
//           is never rewritten: Y = X' * c_j * r_i with the channel / token
//           reciprocals c, r (the exact power-of-two renormalization of
//           (C, R) runs after every second iteration and after the last:
//           the same final (C, R) as renormalizing after every one)
//   RTN     from D1: per-token min / max, codes, packing (K token-major, V in
//           the decode lane order), fp16 metadata and C slices into a staging
//           copy of the group's 8 pages, written out with cp.async.bulk.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cfloat>

#include "kvq_device.cuh"

namespace kvq {

namespace {

constexpr int kMathThreads = 256;       // 8 math warps: warps w and w+4 share TMEM lane quadrant w, split the columns
constexpr int kQThreads = kMathThreads + 32;  // + 1 producer warp (metadata, TMA, MMA) in the quantize kernel
constexpr int kRows = 128;                 // token rows per MMA group
constexpr int kMaxPageBytes = 2048 + 64 + 128;  // 8-bit codes, T = 32
constexpr int kStageBytes = 8 * kMaxPageBytes;  // the group's 8 pages
constexpr long long kWaitNs = 2000000000LL;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kOffH = 0;                   // +-1 Sylvester matrix, 2 x 16 KB SW128 K-major halves
constexpr int kOffX = 32768;               // the group's rows, same layout
constexpr int kOffStage = 65536;           // 2 staging buffers
constexpr int kOffRr = kOffStage + 2 * kStageBytes;   // float r[128]  (token reciprocals)
constexpr int kOffCc = kOffRr + 512;                  // float c[2][4][128] (channel reciprocals per tile, ping-pong)
constexpr int kOffRed = kOffCc + 4096;                // float [8 warps][4 tiles] partial maxima
constexpr int kOffXs = kOffRed + 128;                 // float4 [256] partial statistics exchange
constexpr int kOffMeta = kOffXs + 4096;               // 2 x GroupMeta
constexpr int kOffBar = kOffMeta + 512;               // tma, full, empty, meta[2] mbarriers
constexpr int kOffTmem = kOffBar + 48;
constexpr int kSmemUsed = kOffTmem + 16;
constexpr int kSmemBytes = kSmemUsed + 1024;          // + alignment slack

struct GroupMeta {
  int valid[4];          // tile of the group present and in range
  int pages[4][8];       // block ids of each tile's pages
  int nvalid;
};

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ long long gtime() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// a waiting thread may be suspended up to this long per try (it resumes when
// the phase completes)
constexpr uint32_t kSuspendHintNs = 20000;
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  if (mbar_try(bar, parity)) return true;
  const long long t0 = gtime();
  while (!mbar_try(bar, parity))
    if (gtime() - t0 > kWaitNs) return false;
  return true;
}

// element (row r, channel k) of a 128 x 128 fp16 K-major operand in two
// 64-channel halves of 128-byte rows with the 128-byte swizzle
__device__ __forceinline__ uint32_t sw128_off(int r, int k) {
  const int half = k >> 6, c = (k & 63) >> 3, e = k & 7;
  return half * 16384 + r * 128 + ((c ^ (r & 7)) << 4) + e * 2;
}
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFF);  // start address
  d |= static_cast<uint64_t>(1) << 16;                          // leading offset (unused here)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;                  // 8-row groups 1024 B apart
  d |= static_cast<uint64_t>(1) << 46;                          // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                          // 128-byte swizzle
  return d;
}
// kind::f16, fp32 accumulate, fp16 A/B, both K-major, M = N = 128
constexpr uint32_t kIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void mma_f16(uint32_t dtmem, uint64_t da, uint64_t db, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          dtmem),
      "l"(da), "l"(db), "r"(kIdesc), "r"(acc));
}

// 32 consecutive fp32 columns of this thread's TMEM lane.  The wait takes
// the loaded registers as operands, so no use of them can move above it,
// and carries no memory clobber, so ordinary shared-memory loads can.
__device__ __forceinline__ void tmem_ld32(uint32_t addr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
      "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(addr));
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]), "+r"(r[8]),
        "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]),
        "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]),
        "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// barrier of the two warps (w, w + 4) that share TMEM lane quadrant w
__device__ __forceinline__ void pair_sync(int quadrant) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + quadrant) : "memory");
}
// barrier of the 8 math warps (the producer warp never joins it)
__device__ __forceinline__ void math_sync() { asm volatile("bar.sync 15, 256;" ::: "memory"); }
// barrier of the 256 math threads that also returns whether any of them passed true
__device__ __forceinline__ bool math_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, 15, 256, q;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// Scalar helpers for the per-row statistics (not per element).  The
// approximate forms are within 2 ulp; a scale change that small moves a code
// only for values within ~1e-7 of a rounding boundary.
__device__ __forceinline__ float sqrt_fast(float x) {
  float y;
  asm("sqrt.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float div_fast(float a, float b) {  // full range, 2 ulp
  float y;
  asm("div.full.f32 %0, %1, %2;" : "=f"(y) : "f"(a), "f"(b));
  return y;
}
// the exponent frexpf would return, for m >= 0
__device__ __forceinline__ int frexp_exponent(float m) {
  const uint32_t be = __float_as_uint(m) >> 23;
  if (be - 1u < 254u) return static_cast<int>(be) - 126;  // normal
  int e;
  frexpf(m, &e);  // zero, subnormal, inf, nan
  return e;
}
// ldexpf(x, k): one exact multiply when 2^k is a normal float
__device__ __forceinline__ float scale_pow2(float x, int k) {
  if (k >= -126 && k <= 127) return x * __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
  return ldexpf(x, k);
}

__device__ __forceinline__ float min3f(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// Shifted sums of 32 values x_k * w_k - shift with packed f32x2 arithmetic
// (kChains independent accumulator chains per statistic).
constexpr int kChains = 2;
__device__ __forceinline__ void shifted_sums(const float* x, const float* w, float shift, float2 (&s1)[kChains],
                                             float2 (&s2)[kChains]) {
  const float2 nk = make_float2(-shift, -shift);
#pragma unroll
  for (int k = 0; k < 32; k += 2 * kChains) {
    float2 d[kChains];
#pragma unroll
    for (int c = 0; c < kChains; c += 2) {
      const float4 wv = *reinterpret_cast<const float4*>(w + k + 2 * c);
      d[c] = __ffma2_rn(make_float2(x[k + 2 * c], x[k + 2 * c + 1]), make_float2(wv.x, wv.y), nk);
      d[c + 1] = __ffma2_rn(make_float2(x[k + 2 * c + 2], x[k + 2 * c + 3]), make_float2(wv.z, wv.w), nk);
    }
#pragma unroll
    for (int c = 0; c < kChains; ++c) s1[c] = __fadd2_rn(s1[c], d[c]);
#pragma unroll
    for (int c = 0; c < kChains; ++c) s2[c] = __ffma2_rn(d[c], d[c], s2[c]);
  }
}

__device__ __forceinline__ float2 sum_chains(const float2 (&s)[kChains]) {
  float2 v[kChains];
#pragma unroll
  for (int c = 0; c < kChains; ++c) v[c] = s[c];
#pragma unroll
  for (int h = kChains / 2; h > 0; h >>= 1)
#pragma unroll
    for (int c = 0; c < h; ++c) v[c] = __fadd2_rn(v[c], v[c + h]);
  return v[0];
}

// (mean, M2) of n values from shifted sums (shift k): mean = k + S1/n, M2 = S2 - S1^2/n
struct Moments {
  float mean, m2;
};
__device__ __forceinline__ Moments moments(const float2 (&s1)[kChains], const float2 (&s2)[kChains], float shift,
                                           float n) {
  const float2 a2 = sum_chains(s1);
  const float2 q2 = sum_chains(s2);
  const float a = a2.x + a2.y, q = q2.x + q2.y;
  Moments m;
  m.mean = shift + a / n;
  m.m2 = fmaxf(q - a * (a / n), 0.f);
  return m;
}
// two halves of n values each (always combined in the order (first, second))
__device__ __forceinline__ float combined_std(Moments a, Moments b, float n) {
  const float dm = a.mean - b.mean;
  return sqrt_fast((a.m2 + b.m2 + dm * dm * (0.5f * n)) * (0.5f / n));
}

// Everything after the group's rows are in shared memory and the MMAs are
// done: normalization, RTN, packing into the staging pages, page stores.
// 256 threads: quadrant qd = warp % 4 owns TMEM lanes 32qd..32qd+31 (token
// rows of D1, channel rows of D2); half hf = warp / 4 owns columns
// 64hf..64hf+63 of those rows.  Row statistics that span both halves are
// combined through shared memory (thread tid and its partner tid ^ 128).
// The group: `valid` has bit t set for each present tile t; `store_blk` is,
// for thread q < 8, the block of page q of the group; once the last TMEM
// read is done, one lane per warp arrives on `empty_bar` (0: none).
template <int T, int bits, bool is_v>
__device__ void quantize_group_from_tmem(unsigned char* smem, uint32_t tbase, int valid, int store_blk,
                                         uint32_t empty_bar, const PoolGeom g, int iters, float eps,
                                         unsigned char* stage, uint8_t* pool, int num_heads, int head) {
  constexpr int G = kRows / T;                 // tiles in the group
  constexpr int kPagesPerTile = T / kPageTokens;
  constexpr int kLocal = T <= 64 ? 64 / T : 1; // whole tiles inside my 64 token columns (T <= 64)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int qd = warp & 3, hf = warp >> 2;
  const int row = 32 * qd + lane;             // token of D1 / channel of D2
  float* rr = reinterpret_cast<float*>(smem + kOffRr);
  // c_j per tile in two buffers: iteration `it` reads and updates buffer it&1
  // and writes the renormalized values into the other one
  float* cc_buf = reinterpret_cast<float*>(smem + kOffCc);  // [2][G][128]
  float* cc = cc_buf;
  float* red = reinterpret_cast<float*>(smem + kOffRed);
  float4* xs = reinterpret_cast<float4*>(smem + kOffXs);
  const uint32_t lane_addr = tbase + (static_cast<uint32_t>(32 * qd) << 16);
  const uint32_t d1 = lane_addr + 64 * hf;        // channels 64hf.. of token `row`
  const uint32_t d2 = lane_addr + 128 + 64 * hf;  // tokens 64hf.. of channel `row`
  const int my_tile = row / T;                    // tile of token `row`
  const bool tok_live = (valid >> my_tile) & 1;
  // tiles whose channel statistics this thread computes: T=32 -> 2hf, 2hf+1; T=64 -> hf; T=128 -> 0
  auto ch_tile = [&](int lt) { return T == 128 ? 0 : hf * kLocal + lt; };

  float Cj[kLocal];
#pragma unroll
  for (int lt = 0; lt < kLocal; ++lt) {
    Cj[lt] = 1.f;
    cc[ch_tile(lt) * kRows + row] = 1.f / kSqrtHeadDim;  // c_j = 1 / (sqrt(d) C_j)
  }
  float Ri = 1.f;
  if (hf == 0) rr[row] = 1.f;
  math_sync();

  auto tile_exp = [&](int t) {  // exponent of the tile's max C over the warps that hold it
    float m = 0.f;
    if constexpr (T == 128) {
#pragma unroll
      for (int w = 0; w < 8; ++w) m = fmaxf(m, red[w * 4]);
    } else {  // tile t lives in the token columns of half t / kLocal: warps 4h..4h+3
      const float* rw = red + 16 * (t / kLocal) + t;
      m = fmaxf(fmaxf(rw[0], rw[4]), fmaxf(rw[8], rw[12]));
    }
    return frexp_exponent(m);
  };
  // The (C, R) renormalization by a power of two leaves Y, every std and every
  // clamp decision unchanged, so it runs after every second iteration and
  // after the last: the final (C, R) are those of renormalizing after every
  // iteration (both have max C in [1, 2) and differ from the unrenormalized
  // pair by exact powers of two).  Two iterations move c by at most eps^-2 =
  // 1e12, so the squared deviations of x c stay below 1e36 even for a tile of
  // identical tokens at the fp16 range (three would overflow).  cur: the
  // buffer of c this iteration reads.
  int cur = 0;
  for (int it = 0; it < iters; ++it) {
    const bool renorm = it == iters - 1 || (it & 1) == 1;  // uniform
    cc = cc_buf + cur * (4 * kRows);
    float* cc_next = cc_buf + (cur ^ 1) * (4 * kRows);
    // ---- channel step: channel `row`, token columns 64hf..64hf+63.  The new
    // c_j are published with the per-warp maxima of C for the renormalization.
    if constexpr (T <= 64) {
#pragma unroll
      for (int lt = 0; lt < kLocal; ++lt) {
        const int t = ch_tile(lt);
        if (!((valid >> t) & 1)) continue;
        float2 s1[kChains], s2[kChains];
#pragma unroll
        for (int c = 0; c < kChains; ++c) s1[c] = s2[c] = make_float2(0.f, 0.f);
        float shift = 0.f;
#pragma unroll
        for (int ch = 0; ch < T / 32; ++ch) {
          float x[32];
          tmem_ld32(d2 + lt * T + ch * 32, x);
          if (ch == 0) shift = x[0] * rr[t * T];
          shifted_sums(x, rr + t * T + ch * 32, shift, s1, s2);
        }
        const Moments mo = moments(s1, s2, shift, static_cast<float>(T));
        const float c = cc[t * kRows + row];
        const float sigma = fmaxf(c * sqrt_fast(mo.m2 * (1.f / static_cast<float>(T))), eps);
        Cj[lt] *= sigma;
        cc[t * kRows + row] = fminf(div_fast(c, sigma), FLT_MAX);  // a zero channel keeps a finite factor
      }
    } else {
      float2 s1[kChains], s2[kChains];
#pragma unroll
      for (int c = 0; c < kChains; ++c) s1[c] = s2[c] = make_float2(0.f, 0.f);
      float shift = 0.f;
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        float x[32];
        tmem_ld32(d2 + ch * 32, x);
        if (ch == 0) shift = x[0] * rr[64 * hf];
        shifted_sums(x, rr + 64 * hf + ch * 32, shift, s1, s2);
      }
      const Moments mo = moments(s1, s2, shift, 64.f);
      xs[tid] = make_float4(mo.mean, mo.m2, 0.f, 0.f);
      pair_sync(qd);
      const float4 o = xs[tid ^ 128];
      const Moments other = {o.x, o.y};
      const float sd = hf == 0 ? combined_std(mo, other, 64.f) : combined_std(other, mo, 64.f);
      const float c = cc[row];
      const float sigma = fmaxf(c * sd, eps);
      Cj[0] *= sigma;
      pair_sync(qd);  // both halves have read cc[row]
      if (hf == 0) cc[row] = fminf(div_fast(c, sigma), FLT_MAX);
    }
    if (renorm) {
#pragma unroll
      for (int lt = 0; lt < kLocal; ++lt) {
        // C_j > 0: the float order is the order of the bit patterns
        const float m = __uint_as_float(__reduce_max_sync(kFull, __float_as_uint(Cj[lt])));
        if (lane == 0) red[warp * 4 + ch_tile(lt)] = m;
      }
    }
    math_sync();
    // ---- token step with this iteration's c (before the renormalization,
    // which leaves Y = X' c r unchanged)
    float r_new = 0.f;
    {
      Moments mo = {0.f, 0.f};
      const float r = rr[row];  // read before the pair barrier: the owner rewrites it below
      if (tok_live) {
        float2 s1[kChains], s2[kChains];
#pragma unroll
        for (int c = 0; c < kChains; ++c) s1[c] = s2[c] = make_float2(0.f, 0.f);
        const float* cvec = cc + my_tile * kRows + 64 * hf;
        float shift = 0.f;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
          float x[32];
          tmem_ld32(d1 + ch * 32, x);
          if (ch == 0) shift = x[0] * cvec[0];
          shifted_sums(x, cvec + ch * 32, shift, s1, s2);
        }
        mo = moments(s1, s2, shift, 64.f);
      }
      xs[tid] = make_float4(mo.mean, mo.m2, 0.f, 0.f);
      pair_sync(qd);
      if (tok_live) {
        const float4 o = xs[tid ^ 128];
        const Moments other = {o.x, o.y};
        const float sd = hf == 0 ? combined_std(mo, other, 64.f) : combined_std(other, mo, 64.f);
        const float rho = fmaxf(r * sd, eps);
        Ri *= rho;
        r_new = fminf(div_fast(r, rho), FLT_MAX);  // a zero token keeps a finite factor
      }
    }
    if (!renorm) {  // c stays in this buffer; the new r replaces the old after the pair barrier
      if (tok_live && hf == 0) rr[row] = r_new;
      math_sync();
      continue;
    }
    // ---- (C, R) -> (C / 2^k, R 2^k) per tile, max C in [1, 2): every thread
    // rescales what it owns; cc and rr are read again only after the barrier
    // (the exponent of the token's tile is reused when that tile is one of
    // the channel tiles just handled: warp-uniform, T = 128 always)
    int e_my = 0;
    bool have_my = false;
#pragma unroll
    for (int lt = 0; lt < kLocal; ++lt) {
      const int t = ch_tile(lt);
      const int e = tile_exp(t);
      if (t == my_tile) {
        e_my = e;
        have_my = true;
      }
      Cj[lt] = scale_pow2(Cj[lt], 1 - e);
      if (T < 128 || hf == 0) cc_next[t * kRows + row] = fminf(scale_pow2(cc[t * kRows + row], e - 1), FLT_MAX);
    }
    {
      const int e = have_my ? e_my : tile_exp(my_tile);
      Ri = scale_pow2(Ri, e - 1);
      if (tok_live && hf == 0) rr[row] = fminf(scale_pow2(r_new, 1 - e), FLT_MAX);
    }
    cur ^= 1;
    math_sync();
  }

  // ---- RTN on D1: token `row`, channels 64hf..64hf+63
  cc = cc_buf + cur * (4 * kRows);
  constexpr int qmax = (1 << bits) - 1;
  constexpr bool kGrouped = is_v && bits != 3;  // V in the decode lane order
  const int local = row % T, page_in_tile = local / kPageTokens, p = local % kPageTokens;
  unsigned char* page = stage + (my_tile * kPagesPerTile + page_in_tile) * g.page_bytes;
  const float* cvec = cc + my_tile * kRows + 64 * hf;
  float zu = INFINITY, mu = -INFINITY;
  if (tok_live) {  // pass 1: min / max of u_j = x_j c_j
#pragma unroll
    for (int ch = 0; ch < 2; ++ch) {
      float x[32];
      tmem_ld32(d1 + ch * 32, x);
#pragma unroll
      for (int k = 0; k < 32; k += 4) {
        const float4 cv = *reinterpret_cast<const float4*>(cvec + ch * 32 + k);
        const float2 u0 = __fmul2_rn(make_float2(x[k], x[k + 1]), make_float2(cv.x, cv.y));
        const float2 u1 = __fmul2_rn(make_float2(x[k + 2], x[k + 3]), make_float2(cv.z, cv.w));
        zu = min3f(zu, u0.x, u0.y);
        zu = min3f(zu, u1.x, u1.y);
        mu = max3f(mu, u0.x, u0.y);
        mu = max3f(mu, u1.x, u1.y);
      }
    }
  }
  xs[tid] = make_float4(zu, mu, 0.f, 0.f);
  pair_sync(qd);
  if (tok_live) {
    const float4 o = xs[tid ^ 128];
    zu = fminf(zu, o.x);
    mu = fmaxf(mu, o.y);
    const float r = rr[row];
    const float z = zu * r, mx = mu * r;
    const float s = div_fast(mx - z, static_cast<float>(qmax));
    const float a = s > 0.f ? div_fast(r, s) : 0.f;  // s == 0: every code is 0
    const float b0 = -zu * a;
    // q = t + 1.5 * 2^23 holds round_half_even(t) in its low mantissa bits,
    // so its bit pattern is 0x4B400000 + code.  Words are built by shift-adds
    // of the bit patterns and one subtraction of the shifted constants
    // (arithmetic mod 2^32); codes lie in [0, 2^b - 1] because min and max of
    // the row map to 0 and 2^b - 1 by construction.
    constexpr uint32_t kMagicBits = 0x4B400000u;
    const float2 a2 = make_float2(a, a), b2 = make_float2(b0, b0);
    const float2 magic2 = make_float2(12582912.0f, 12582912.0f);  // 1.5 * 2^23
    if constexpr (!kGrouped) {
      uint32_t words[2 * bits];  // channels 64hf..64hf+63: 2b words
#pragma unroll
      for (int w = 0; w < 2 * bits; ++w) words[w] = 0u;
      float x[32];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        if ((c & 31) == 0) {  // pass 2 for the next 32 channels: u_j = x_j c_j, then u_j a + b0 + magic
          tmem_ld32(d1 + c, x);
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            const float4 cv = *reinterpret_cast<const float4*>(cvec + c + k);
            const float2 u0 = __fmul2_rn(make_float2(x[k], x[k + 1]), make_float2(cv.x, cv.y));
            const float2 u1 = __fmul2_rn(make_float2(x[k + 2], x[k + 3]), make_float2(cv.z, cv.w));
            const float2 q0 = __fadd2_rn(__ffma2_rn(u0, a2, b2), magic2);
            const float2 q1 = __fadd2_rn(__ffma2_rn(u1, a2, b2), magic2);
            x[k] = q0.x; x[k + 1] = q0.y; x[k + 2] = q1.x; x[k + 3] = q1.y;
          }
        }
        const uint32_t qb = __float_as_uint(x[c & 31]);
        const int bit = c * bits;
        if constexpr (bits == 3) {
          const uint32_t code = (qb - kMagicBits) & 7u;
          words[bit >> 5] |= code << (bit & 31);
          if ((bit & 31) + 3 > 32) words[(bit >> 5) + 1] |= code >> (32 - (bit & 31));
        } else {
          words[bit >> 5] += qb << (bit & 31);
        }
      }
      if constexpr (bits != 3) {
        uint32_t k0 = 0;  // the magic constant shifted into every field of a word
#pragma unroll
        for (int f = 0; f < 32 / bits; ++f) k0 += kMagicBits << (bits * f);
#pragma unroll
        for (int w = 0; w < 2 * bits; ++w) words[w] -= k0;
      }
      unsigned char* rec = page + p * (kHeadDim * bits / 8) + hf * (8 * bits);
      if constexpr (bits == 3) {  // 24 bytes per half at an 8-byte aligned offset
#pragma unroll
        for (int w = 0; w < 3; ++w) reinterpret_cast<uint2*>(rec)[w] = make_uint2(words[2 * w], words[2 * w + 1]);
      } else {
#pragma unroll
        for (int w = 0; w < bits / 2; ++w)
          reinterpret_cast<uint4*>(rec)[w] = make_uint4(words[4 * w], words[4 * w + 1], words[4 * w + 2], words[4 * w + 3]);
      }
    } else {
      // channels c = 8n + g8 with n in [8hf, 8hf+8): half-word per (g8, m), m = n / (16 / bits)
      constexpr int h = 16 / bits;          // code pairs per word
      constexpr int nm = 8 / h;             // m values in my half: 2 (b=4) or 1 (b=2)
      uint32_t hw[8 * nm];
#pragma unroll
      for (int w = 0; w < 8 * nm; ++w) hw[w] = 0u;
      float x[32];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        if ((c & 31) == 0) {  // pass 2 for the next 32 channels: u_j = x_j c_j, then u_j a + b0 + magic
          tmem_ld32(d1 + c, x);
#pragma unroll
          for (int k = 0; k < 32; k += 4) {
            const float4 cv = *reinterpret_cast<const float4*>(cvec + c + k);
            const float2 u0 = __fmul2_rn(make_float2(x[k], x[k + 1]), make_float2(cv.x, cv.y));
            const float2 u1 = __fmul2_rn(make_float2(x[k + 2], x[k + 3]), make_float2(cv.z, cv.w));
            const float2 q0 = __fadd2_rn(__ffma2_rn(u0, a2, b2), magic2);
            const float2 q1 = __fadd2_rn(__ffma2_rn(u1, a2, b2), magic2);
            x[k] = q0.x; x[k + 1] = q0.y; x[k + 2] = q1.x; x[k + 3] = q1.y;
          }
        }
        const uint32_t qb = __float_as_uint(x[c & 31]);
        // n = 8 hf + c / 8 and 8 hf is a multiple of h, so m and e depend on c
        // alone: compile-time register indices after unrolling
        const int q8 = c >> 3, g8 = c & 7;
        const int m = q8 / h, e = q8 % h;
        hw[g8 * nm + m] += qb << (bits * e);
      }
      uint32_t k0 = 0;
#pragma unroll
      for (int f = 0; f < h; ++f) k0 += kMagicBits << (bits * f);
      // word (lane L = 4*g8 + t, k = 2m + u) = low half from the even token of
      // the pair {2t + 8u, 2t + 8u + 1}, high half from the odd token
      const int t4 = (p & 7) >> 1, u = p >> 3, odd = p & 1;
      // low halves of (mine, other) in token order: bytes 0,1 of the even
      // token's value, then bytes 0,1 of the odd token's
      const uint32_t order = odd ? 0x1054u : 0x5410u;
#pragma unroll
      for (int idx = 0; idx < 8 * nm; ++idx) {
        const uint32_t mine = hw[idx] - k0;  // its low 16 bits hold the fields
        const uint32_t other = __shfl_xor_sync(kFull, mine, 1);
        const int g8 = idx / nm, m = hf * nm + idx % nm;
        if ((g8 & 1) == odd) {  // the pair's two tokens split the words
          const uint32_t word = __byte_perm(mine, other, order);
          const int L = 4 * g8 + t4, kk = 2 * m + u;
          *reinterpret_cast<uint32_t*>(page + ((kk >> 2) * 32 + L) * 16 + (kk & 3) * 4) = word;
        }
      }
    }
    if (hf == 0)
      *reinterpret_cast<__half2*>(page + g.meta_off + 4 * p) =
          __halves2half2(__float2half_rn(s * Ri), __float2half_rn(z * Ri));
  }
  // every TMEM read of this group is done: the producer may overwrite it
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncwarp();
  if (empty_bar != 0 && lane == 0)
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(empty_bar) : "memory");
  // C slices: channel thread `row` writes C~ of its tiles into page k = row / cs of the tile
#pragma unroll
  for (int lt = 0; lt < kLocal; ++lt) {
    const int t = ch_tile(lt);
    if (!((valid >> t) & 1) || (T == 128 && hf != 0)) continue;
    const int pg = row / g.cs_channels;
    *reinterpret_cast<__half*>(stage + (t * kPagesPerTile + pg) * g.page_bytes + g.cslice_off +
                               2 * (row % g.cs_channels)) = __float2half_rn(Cj[lt]);
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  math_sync();
  // page stores: thread q < 8 stores page q of the group
  if (tid < 8) {
    const int t = tid / kPagesPerTile;
    if (t < G && ((valid >> t) & 1)) {
      const int blk = store_blk;
      uint8_t* dst = pool + (static_cast<size_t>(blk) * num_heads + head) * static_cast<size_t>(g.page_bytes);
      asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                   "r"(smem_u32(stage + tid * g.page_bytes)), "r"(g.page_bytes)
                   : "memory");
    }
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  }
}

// the group function for this item's code width and K|V
template <int T, int BK, int BV>
__device__ __forceinline__ void quantize_group_dispatch(unsigned char* smem, uint32_t tbase, int valid, int store_blk,
                                                        uint32_t empty_bar, bool is_v, const PoolGeom g, int iters,
                                                        float eps, unsigned char* stage, uint8_t* pool, int num_heads,
                                                        int head) {
  if (is_v)
    quantize_group_from_tmem<T, BV, true>(smem, tbase, valid, store_blk, empty_bar, g, iters, eps, stage, pool,
                                          num_heads, head);
  else
    quantize_group_from_tmem<T, BK, false>(smem, tbase, valid, store_blk, empty_bar, g, iters, eps, stage, pool,
                                           num_heads, head);
}

// The +-1 matrix M[r][k] = s_k (-1)^popcount(r & k) in the operand layout.
// It is B of D1 = X M^T = X D_s H and A of D2 = M X^T = H D_s X^T (H is
// symmetric), so one copy serves both layouts; s = 1 for the plain rotation.
__device__ void build_h(unsigned char* smem, uint32_t seed) {
  for (int idx = threadIdx.x; idx < kRows * kHeadDim; idx += blockDim.x) {
    const int r = idx >> 7, k = idx & 127;
    const float h = (__popc(r & k) & 1) ? -1.f : 1.f;
    *reinterpret_cast<__half*>(smem + kOffH + sw128_off(r, k)) = __float2half_rn(h * rotation_sign(seed, k));
  }
}

__device__ uint32_t tmem_alloc(unsigned char* smem) {
  uint32_t* slot = reinterpret_cast<uint32_t*>(smem + kOffTmem);
  if ((threadIdx.x >> 5) == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)), "r"(256));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  return *slot;
}

__device__ void tmem_free(uint32_t tbase) {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if ((threadIdx.x >> 5) == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(256));
}

// one thread: the 16 MMAs of a group (the caller commits)
__device__ void issue_mmas_nocommit(unsigned char* smem, uint32_t tbase) {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t sx = smem_u32(smem + kOffX), sh = smem_u32(smem + kOffH);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint32_t koff = (s >> 2) * 16384 + (s & 3) * 32;
    mma_f16(tbase, sw128_desc(sx + koff), sw128_desc(sh + koff), s > 0);          // D1 = X H
    mma_f16(tbase + 128, sw128_desc(sh + koff), sw128_desc(sx + koff), s > 0);    // D2 = H X^T
  }
}

// one thread: the 16 MMAs of a group, completion on mma_bar
__device__ void issue_mmas(unsigned char* smem, uint32_t tbase, uint32_t mma_bar) {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t sx = smem_u32(smem + kOffX), sh = smem_u32(smem + kOffH);
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    const uint32_t koff = (s >> 2) * 16384 + (s & 3) * 32;
    mma_f16(tbase, sw128_desc(sx + koff), sw128_desc(sh + koff), s > 0);          // D1 = X H
    mma_f16(tbase + 128, sw128_desc(sh + koff), sw128_desc(sx + koff), s > 0);    // D2 = H X^T
  }
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mma_bar)
               : "memory");
}

struct QuantTcArgs {
  QuantizeArgs a;
  int num_items;  // groups x heads x 2
  int groups;
};

// true when this CTA's k-th item exists (the producer left its loop early)
__device__ __forceinline__ bool item_left(const QuantTcArgs& qa, int k) {
  return blockIdx.x + static_cast<long long>(k) * gridDim.x < qa.num_items;
}

// thread 0: validate the group's tiles, fill its metadata slot and issue the
// TMA loads of its valid tiles; returns the number of valid tiles.
template <int T>
__device__ int prepare_group(const QuantTcArgs& qa, const CUtensorMap* tmk, const CUtensorMap* tmv, int item,
                             GroupMeta* gm, unsigned char* smem, uint32_t tma_bar) {
  constexpr int G = kRows / T;
  constexpr int kPagesPerTile = T / kPageTokens;
  const QuantizeArgs& a = qa.a;
  const int kv = item & 1, head = (item >> 1) % a.cfg.num_kv_heads, grp = (item >> 1) / a.cfg.num_kv_heads;
  const void* src = kv ? a.src_v : a.src_k;
  int nvalid = 0;
  for (int t = 0; t < G; ++t) {
    const int tile = grp * G + t;
    bool ok = src != nullptr && tile < a.num_tiles;
    int src_row = 0, seq = 0, tidx = 0;
    if (ok) {
      src_row = a.tile_desc[3 * tile];
      seq = a.tile_desc[3 * tile + 1];
      tidx = a.tile_desc[3 * tile + 2];
      bool good = src_row >= 0 && src_row <= a.num_rows - T && seq >= 0 && seq < a.num_seqs && tidx >= 0 &&
                  (tidx + 1) * kPagesPerTile <= a.max_blocks_per_seq;
      for (int k = 0; good && k < kPagesPerTile; ++k) {
        const int blk = a.block_tables[static_cast<size_t>(seq) * a.max_blocks_per_seq + tidx * kPagesPerTile + k];
        good = blk >= 0 && blk < a.num_blocks;
        gm->pages[t][k] = blk;
      }
      if (!good && head == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
      ok = good;
    }
    gm->valid[t] = ok;
    nvalid += ok;
  }
  gm->nvalid = nvalid;
  if (nvalid > 0) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(tma_bar), "r"(nvalid * T * 256)
                 : "memory");
    const CUtensorMap* tm = kv ? tmv : tmk;
    for (int t = 0; t < G; ++t) {
      if (!gm->valid[t]) continue;
      const int src_row = a.tile_desc[3 * (grp * G + t)];
      for (int half = 0; half < 2; ++half) {
        const uint32_t dst = smem_u32(smem + kOffX + half * 16384 + t * T * 128);
        asm volatile(
            "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
            "%4}], [%5];" ::"r"(dst),
            "l"(reinterpret_cast<uint64_t>(tm)), "r"(64 * half), "r"(head), "r"(src_row), "r"(tma_bar)
            : "memory");
      }
    }
  }
  return nvalid;
}

template <int T, int BK, int BV>
__global__ void __launch_bounds__(kQThreads, 2) quantize_tc_kernel(const __grid_constant__ CUtensorMap tmk,
                                                    const __grid_constant__ CUtensorMap tmv, QuantTcArgs qa) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  constexpr int G = kRows / T;
  constexpr int kPagesPerTile = T / kPageTokens;
  const QuantizeArgs& a = qa.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  GroupMeta* meta = reinterpret_cast<GroupMeta*>(smem + kOffMeta);
  // tma: rows landed (producer only); full: the group's MMAs are done (TMEM
  // holds it, rows buffer free); empty: the 8 math warps finished reading
  // TMEM; meta[2]: a group's metadata slot is written
  const uint32_t tma_bar = smem_u32(smem + kOffBar), full_bar = tma_bar + 8, empty_bar = tma_bar + 16;
  const uint32_t meta_bar0 = tma_bar + 24;

  build_h(smem, a.cfg.rotation_seed);
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(tma_bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(full_bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 8;" ::"r"(empty_bar));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(meta_bar0));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(meta_bar0 + 8));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  const uint32_t tbase = tmem_alloc(smem);  // includes a __syncthreads

  if (warp == kMathThreads / 32) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t tma_phase = 0;
      int k = 0;
      bool tma_pending = false;
      for (int item = blockIdx.x; item < qa.num_items; item += gridDim.x, ++k) {
        const int slot = k & 1;
        if (k > 0 && !mbar_wait(full_bar, (k - 1) & 1)) break;  // previous MMAs done: rows buffer free
        const int nvalid = prepare_group<T>(qa, &tmk, &tmv, item, &meta[slot], smem, tma_bar);
        asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(meta_bar0 + 8 * slot) : "memory");
        if (nvalid > 0) {
          tma_pending = true;
          if (!mbar_wait(tma_bar, tma_phase)) break;
          tma_pending = false;
          tma_phase ^= 1u;
        }
        if (k > 0 && !mbar_wait(empty_bar, (k - 1) & 1)) break;  // math warps done with the previous TMEM
        if (nvalid > 0) {
          issue_mmas_nocommit(smem, tbase);
          asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(full_bar)
                       : "memory");
        } else {  // nothing to compute: the previous MMAs were already waited for
          asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(full_bar) : "memory");
        }
      }
      if (item_left(qa, k)) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
      if (tma_pending) (void)mbar_wait(tma_bar, tma_phase);  // a load still in flight must land first
      if (k > 0) (void)mbar_wait(full_bar, (k - 1) & 1);    // and the last MMAs must be done
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ math warps
    int k = 0;
    for (int item = blockIdx.x; item < qa.num_items; item += gridDim.x, ++k) {
      const int slot = k & 1;
      bool ok = mbar_wait(meta_bar0 + 8 * slot, (k >> 1) & 1);
      const GroupMeta& gm = meta[slot];
      int valid = 0, store_blk = 0;
      if (ok) {
        for (int t = 0; t < G; ++t) valid |= (gm.valid[t] ? 1 : 0) << t;
        if (tid < 8 && tid / kPagesPerTile < G && ((valid >> (tid / kPagesPerTile)) & 1))
          store_blk = gm.pages[tid / kPagesPerTile][tid % kPagesPerTile];
        ok = mbar_wait(full_bar, k & 1);
      }
      if (math_any(!ok)) {  // one decision for all math threads
        if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
        break;
      }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const int kv = item & 1, head = (item >> 1) % a.cfg.num_kv_heads;
      if (valid != 0) {
        // the staging buffer used two groups ago must have been read by its stores
        if (tid < 8) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        math_sync();
        const PoolGeom g = kv ? a.gv : a.gk;
        unsigned char* stage = smem + kOffStage + (k & 1) * kStageBytes;
        quantize_group_dispatch<T, BK, BV>(smem, tbase, valid, store_blk, empty_bar, kv != 0, g, a.cfg.iters,
                                           a.cfg.std_eps, stage, static_cast<uint8_t*>(kv ? a.v_pool : a.k_pool),
                                           a.cfg.num_kv_heads, head);
      } else {
        if (tid < 8) asm volatile("cp.async.bulk.commit_group;" ::: "memory");  // keeps one group per item
        __syncwarp();
        if (lane == 0) asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(empty_bar) : "memory");
      }
    }
    if (tid < 8) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
  }
  tmem_free(tbase);  // includes a __syncthreads of all warps
}

// ---------------------------------------------------------------- self-test
// One thread waits, with the kernels' bounded wait, on a barrier that nothing
// arrives at; the wait gives up after its limit and the timeout is recorded.
__global__ void selftest_wait_kernel(int32_t* dev_status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if (!mbar_wait(b, 0)) report_error(dev_status, KVQ_ERR_DEVICE_TIMEOUT);
}

// ---------------------------------------------------------------- append
// One CTA per (sequence, KV head, K|V): every tile completed by the new
// tokens is loaded (old tail rows + new rows) into the same swizzled layout
// and quantized by the same code path as kvq_quantize_tiles (bit-identical
// pages); the remaining new tokens go to the fp16 tail.
template <int T, int BK, int BV>
__global__ void __launch_bounds__(kMathThreads, 2) append_tc_kernel(AppendArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  constexpr int kPagesPerTile = T / kPageTokens;
  const int b = blockIdx.x, head = blockIdx.y, kv = blockIdx.z, tid = threadIdx.x;
  const __half* src = static_cast<const __half*>(kv ? a.new_v : a.new_k);
  __half* tail = static_cast<__half*>(kv ? a.v_tail : a.k_tail);
  if (src == nullptr || tail == nullptr) return;
  const PoolGeom g = kv ? a.gv : a.gk;
  uint8_t* pool = static_cast<uint8_t*>(kv ? a.v_pool : a.k_pool);
  const int nh = a.cfg.num_kv_heads;
  const int l0 = a.seq_lens_before[b];
  const int start = a.cu_new[b];
  const int n = a.cu_new[b + 1] - start;
  if (n <= 0 || l0 < 0) return;
  const int end = l0 + n;
  __half* tail_base = tail + (static_cast<size_t>(b) * nh + head) * T * kHeadDim;
  GroupMeta* gm = reinterpret_cast<GroupMeta*>(smem + kOffMeta);
  const uint32_t mma_bar = smem_u32(smem + kOffBar + 8);
  int* flag = reinterpret_cast<int*>(smem + kOffTmem + 4);

  if (l0 / T < end / T) {  // at least one tile completes: tensor-core set-up
    build_h(smem, a.cfg.rotation_seed);
    for (int i = tid; i < kRows * kHeadDim / 8; i += kMathThreads) {  // rows of the unused tiles: zeros
      const int r = i / 16, c = i % 16;
      if (r >= T) *reinterpret_cast<uint4*>(smem + kOffX + sw128_off(r, c * 8)) = make_uint4(0, 0, 0, 0);
    }
    if (tid == 0) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(mma_bar));
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      *flag = 0;
      gm->valid[1] = gm->valid[2] = gm->valid[3] = 0;
    }
    const uint32_t tbase = tmem_alloc(smem);
    uint32_t mma_phase = 0;
    int iter = 0;
    for (int t = l0 / T; t < end / T; ++t, ++iter) {
      if (tid < kPagesPerTile) {
        const int lb = t * kPagesPerTile + tid;
        const int blk = lb < a.max_blocks_per_seq ? a.block_tables[static_cast<size_t>(b) * a.max_blocks_per_seq + lb]
                                                   : -1;
        gm->pages[0][tid] = blk;
        if (blk < 0 || blk >= a.num_blocks) {
          report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
          *flag = 2;
        }
      }
      // rows of the tile: 16-byte pieces into the swizzled layout
      for (int i = tid; i < T * 16; i += kMathThreads) {
        const int r = i / 16, c = i % 16;
        const int q = t * T + r;
        const __half* row = (q < l0) ? tail_base + static_cast<size_t>(q % T) * kHeadDim
                                     : src + (static_cast<size_t>(start + q - l0) * nh + head) * kHeadDim;
        *reinterpret_cast<uint4*>(smem + kOffX + sw128_off(r, c * 8)) = *reinterpret_cast<const uint4*>(row + c * 8);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncthreads();
      if (*flag == 2) {  // bad page: skip this tile (reported)
        __syncthreads();
        if (tid == 0) *flag = 0;
        __syncthreads();
        continue;
      }
      if (tid == 0) {
        gm->valid[0] = 1;
        gm->nvalid = 1;
        issue_mmas(smem, tbase, mma_bar);
      }
      __syncthreads();
      if (!mbar_wait(mma_bar, mma_phase)) {
        report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
        *flag = 1;
      }
      mma_phase ^= 1u;
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      __syncthreads();
      if (*flag == 1) break;
      if (tid < 8) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
      __syncthreads();
      const int store_blk = tid < kPagesPerTile ? gm->pages[0][tid] : 0;
      quantize_group_dispatch<T, BK, BV>(smem, tbase, 1, store_blk, 0u, kv != 0, g, a.cfg.iters, a.cfg.std_eps,
                                         smem + kOffStage + (iter & 1) * kStageBytes, pool, nh, head);
      asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
      __syncthreads();
    }
    if (tid < 8) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    tmem_free(tbase);
  }
  // remaining tokens of the unfinished tile go to the tail (16-byte pieces)
  const int first = max(l0, (end / T) * T);
  const int count = end - first;
  for (int idx = tid; idx < count * (kHeadDim / 8); idx += kMathThreads) {
    const int r = idx / (kHeadDim / 8), piece = idx % (kHeadDim / 8);
    const int q = first + r;
    const uint4 v = *reinterpret_cast<const uint4*>(
        src + (static_cast<size_t>(start + q - l0) * nh + head) * kHeadDim + 8 * piece);
    *reinterpret_cast<uint4*>(tail_base + static_cast<size_t>(q % T) * kHeadDim + 8 * piece) = v;
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 3-D map over rows [num_rows][H][d] fp16: box (64 channels, 1 head, T rows), 128-byte swizzle
bool make_rows_map(CUtensorMap* m, const void* base, int num_heads, int num_rows, int T) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(kHeadDim), static_cast<cuuint64_t>(num_heads),
                        static_cast<cuuint64_t>(std::max(num_rows, T))};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(kHeadDim) * 2, static_cast<cuuint64_t>(num_heads) * kHeadDim * 2};
  cuuint32_t box[3] = {64, 1, static_cast<cuuint32_t>(T)};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int T, int BK, int BV>
cudaError_t launch_quantize_tc(const QuantizeArgs& a, cudaStream_t s) {
  CUtensorMap mk, mv;
  // a missing source gets the other one's map (its items are never loaded)
  const void* sk = a.src_k ? a.src_k : a.src_v;
  const void* sv = a.src_v ? a.src_v : a.src_k;
  if (!make_rows_map(&mk, sk, a.cfg.num_kv_heads, a.num_rows, T) ||
      !make_rows_map(&mv, sv, a.cfg.num_kv_heads, a.num_rows, T))
    return cudaErrorInvalidValue;
  QuantTcArgs qa;
  qa.a = a;
  qa.groups = (a.num_tiles + kRows / T - 1) / (kRows / T);
  const long long items = static_cast<long long>(qa.groups) * a.cfg.num_kv_heads * 2;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  qa.num_items = static_cast<int>(items);
  auto kern = quantize_tc_kernel<T, BK, BV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // two CTAs per SM: 2 x 256 TMEM columns and 2 x ~89 KB of shared memory
  const int grid = static_cast<int>(std::min<long long>(items, 2LL * sms));
  kern<<<grid, kQThreads, kSmemBytes, s>>>(mk, mv, qa);
  return cudaGetLastError();
}

template <int T, int BK, int BV>
cudaError_t launch_append_tc(const AppendArgs& a, cudaStream_t s) {
  auto kern = append_tc_kernel<T, BK, BV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_seqs, a.cfg.num_kv_heads, 2);
  kern<<<grid, kMathThreads, kSmemBytes, s>>>(a);
  return cudaGetLastError();
}

// (T, b_K, b_V) -> kernel instance
template <template <int, int, int> class L, typename Args>
cudaError_t dispatch_bits(const Args& a, cudaStream_t s) {
  const int bk = a.cfg.bits_k, bv = a.cfg.bits_v;
  switch (a.cfg.tile_tokens) {
#define KVQ_BITS(TT)                                                            \
  case TT:                                                                    \
    if (bk == 4 && bv == 4) return L<TT, 4, 4>::run(a, s);                    \
    if (bk == 4 && bv == 2) return L<TT, 4, 2>::run(a, s);                    \
    if (bk == 4 && bv == 3) return L<TT, 4, 3>::run(a, s);                    \
    if (bk == 2 && bv == 4) return L<TT, 2, 4>::run(a, s);                    \
    if (bk == 2 && bv == 2) return L<TT, 2, 2>::run(a, s);                    \
    if (bk == 2 && bv == 3) return L<TT, 2, 3>::run(a, s);                    \
    if (bk == 3 && bv == 4) return L<TT, 3, 4>::run(a, s);                    \
    if (bk == 3 && bv == 2) return L<TT, 3, 2>::run(a, s);                    \
    if (bk == 8 && bv == 8) return L<TT, 8, 8>::run(a, s);                    \
    return L<TT, 3, 3>::run(a, s);
    KVQ_BITS(32)
    KVQ_BITS(64)
    default:
      KVQ_BITS(128)
#undef KVQ_BITS
  }
}

template <int T, int BK, int BV>
struct QuantizeLauncher {
  static cudaError_t run(const QuantizeArgs& a, cudaStream_t s) { return launch_quantize_tc<T, BK, BV>(a, s); }
};
template <int T, int BK, int BV>
struct AppendLauncher {
  static cudaError_t run(const AppendArgs& a, cudaStream_t s) { return launch_append_tc<T, BK, BV>(a, s); }
};

}  // namespace

cudaError_t launch_selftest_wait_quantize(int32_t* dev_status, cudaStream_t s) {
  selftest_wait_kernel<<<1, 1, 0, s>>>(dev_status);
  return cudaGetLastError();
}

cudaError_t launch_quantize_tiles(const QuantizeArgs& a, cudaStream_t s) {
  if (a.cfg.head_dim != kHeadDim) return launch_generic_quantize(a, s);
  if (a.num_tiles == 0) return cudaSuccess;
  return dispatch_bits<QuantizeLauncher>(a, s);
}

cudaError_t launch_append_tokens(const AppendArgs& a, cudaStream_t s) {
  if (a.cfg.head_dim != kHeadDim) return launch_generic_append(a, s);
  if (a.num_seqs == 0) return cudaSuccess;
  return dispatch_bits<AppendLauncher>(a, s);
}

}  // namespace kvq
