// Read path, chunked prefill: a chunk of n new tokens per sequence attends to
// the quantized cache (pages read directly, never re-materialised as fp16;
// aitrends.kr article 74976, "TL;DR" and glossary "attention backend") and,
// causally, to its own raw fp16 rows.
//
// One kernel, one CTA (8 warps) per (sequence, KV head, 128 query rows).  The
// query rows of a (sequence, KV head) are the chunk tokens x the g query heads
// of that KV head, token-major: row i*g + j is chunk token i, head j.  Warp w
// owns TMEM lanes 32 (w % 4) .. +31 (one query row per thread) and column half
// w / 4 (32 of a block's 64 tokens in the softmax, 64 of the 128 channels in
// the accumulators).  Every contraction runs on the tcgen05 tensor cores (fp16
// operands, K-major with the 128-byte swizzle in shared memory or row-per-lane
// in TMEM; fp32 accumulators in TMEM; one thread issues, a commit to an
// mbarrier signals completion).  fp32 operands enter as hi + lo * 2^-11 fp16
// pairs whose two products accumulate separately (see hi_lo2).
//
// A. Context tiles, rotated domain.  q' = q D_s H (one MMA against H, scaled
//    into the log2 domain, kept in TMEM) and per tile of the context, the
//    decode kernel's algebra:
//      score_i = s~K_i (q'' . codeK_i) + z~K_i sum_j q''_j,   q'' = q' * C~K_t
//      acc'_j += C~V_tj (sum_i p_i s~V_i codeV_ij + sum_i p_i z~V_i)
//    QK (per 64-token block): D_S[128][80] = q''_hi . B_K^T and its lo twin,
//    with q'' built per tile into TMEM as the A operand and B_K = the block's
//    K codes as exact fp16 integers, a row of ones (column 64 is then
//    sum_j q''_j) and zero rows.  PV: D_O[128][128] = P_hi . B_V^T and its lo
//    twin, P = p * s~V, B_V = V codes channel-major (exact).  C~V scales D_O's
//    columns per tile, so D_O is folded into register accumulators block by
//    block.  Tiles are staged whole (K and V pages) by cp.async.bulk, double-
//    buffered; PV runs while the next block's codes are unpacked, and no TMEM
//    load overlaps an MMA that writes TMEM.
// B. Raw keys, original domain: the fp16 tail of the cache, then the chunk's
//    own rows, causal (chunk token i sees tail + chunk rows 0..i).  QK: q
//    (fp16, exact) . K_raw^T; PV: P_hi / P_lo . V_raw^T (V transposed into
//    shared memory).  Separate running max / sum / accumulator; the context
//    accumulator waits in TMEM meanwhile.
// C. The two parts are merged by their log-sum-exp weights; the rotated part
//    (already divided by the softmax sum) is taken back with one MMA against H,
//    then the channel signs and 1/sqrt(d); fp16 output.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "kvq_device.cuh"

namespace kvq {

namespace {

constexpr int kPfThreads = 256;
constexpr int kRows = 128;                  // query rows per CTA (TMEM lanes)
constexpr int kBlk = 64;                    // context tokens per MMA block
constexpr int kNS = kBlk + 16;              // score columns: tokens, sum(q''), zero rows
constexpr long long kWaitNs = 2000000000LL; // bounded waits: 2 s

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kOffAqHi = 0;                        // q''_hi: 128 x 128 fp16, two 16 KB channel atoms
constexpr int kOffAqLo = 32768;                    // q''_lo
constexpr int kOffBk = 65536;                      // B_K: 80 x 128 fp16, two 10 KB channel atoms
constexpr int kBkAtom = kNS * 128;                 // 10240
constexpr int kOffBv = kOffBk + 2 * kBkAtom;       // B_V: 2 buffers of 128 channels x 64 tokens fp16 (16 KB)
constexpr int kOffPHi = kOffBv + 2 * 16384;        // P_hi: 128 rows x 64 tokens fp16
constexpr int kOffPLo = kOffPHi + 16384;           // P_lo
constexpr int kOffRed = kOffPLo + 16384;           // float red[3][2][128]: row max, sum p, sum p z~V
constexpr int kOffF = kOffRed + 3 * 2 * kRows * 4; // 2 x float tile scalars: C~K[128], C~V[128], s~K, z~K, s~V, z~V [128]
constexpr int kFBuf = 6 * 128;                     // floats per scalar buffer
constexpr int kOffBar = kOffF + 2 * kFBuf * 4;     // mbarriers: stage 0, stage 1, mma, qk, pv
constexpr int kOffMisc = kOffBar + 64;             // TMEM slot, flags
constexpr int kOffStage = kOffMisc + 64;
// the set-up rotation borrows B_K .. B_V for H (128 x 128 fp16, 32 KB); the
// final one borrows the two B_V buffers
static_assert(kOffBk + 32768 <= kOffPHi, "H fits in front of P");
static_assert(kOffBv + 32768 <= kOffPHi, "H fits over the B_V buffers");
static_assert(kOffBv % 1024 == 0 && kOffPHi % 1024 == 0 && kOffPLo % 1024 == 0, "atoms 1024-aligned");

template <int T, int BK, int BV>
struct PfGeom {
  static constexpr int kPages = T / kPageTokens;
  static constexpr int kCodesK = kPageTokens * kHeadDim * BK / 8;
  static constexpr int kCodesV = kPageTokens * kHeadDim * BV / 8;
  static constexpr int kCs = kHeadDim * kPageTokens / T;  // channels of C per page
  static constexpr int kCsBytes = (2 * kCs + 15) / 16 * 16;
  static constexpr int kPageK = kCodesK + 64 + kCsBytes;
  static constexpr int kPageV = kCodesV + 64 + kCsBytes;
  static constexpr int kStage = kPages * (kPageK + kPageV);
  static constexpr int kValid = T < kBlk ? T : kBlk;  // tokens per block
  static constexpr int kBlocks = T < kBlk ? 1 : T / kBlk;
  static constexpr int kSmem = kOffStage + 2 * kStage + 1024;  // + alignment slack
  static_assert(kSmem <= 232448, "shared memory per block");
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ long long gtime() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
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
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}
// Order of the channels along the QK contraction: the K codes of a 32-bit
// word (W = 32/b channels, fields in channel order) unpack into pairs
// (field e, field e + W/2), so MMA position 2e + s of the word's group holds
// channel e + s W/2.  q'' is written in the same order (the dot product does
// not care which order, only that both operands share it).
// At 3 bits the codes are extracted one by one and the order is the
// natural one (position k holds channel k).
template <int B>
__device__ __forceinline__ constexpr int qk_channel(int kpos) {
  if (B == 3) return kpos;
  constexpr int W = 32 / (B == 3 ? 4 : B);
  const int p = kpos % W;
  return kpos - p + (p >> 1) + (p & 1) * (W / 2);
}

// b-bit field at bit `bit` of a little-endian run of 32-bit words (b <= 8)
template <int B>
__device__ __forceinline__ uint32_t field_at(const uint32_t* w, int bit) {
  return __funnelshift_r(w[bit >> 5], w[(bit >> 5) + 1], bit & 31) & ((1u << B) - 1u);
}
// two codes as an fp16 pair of exact small integers (low half `lo`)
__device__ __forceinline__ uint32_t code_pair_f16(uint32_t lo, uint32_t hi) {
  return h2_as_u32(__hsub2(u32_as_h2(lo | (hi << 16) | 0x64006400u), __float2half2_rn(1024.f)));
}

// Byte offset of (row r, position k) in a K-major fp16 operand of `rows` rows
// stored as 64-element atoms of 128-byte rows with the 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_off(int r, int k, int rows) {
  return (k >> 6) * rows * 128 + r * 128 + ((((k & 63) >> 3) ^ (r & 7)) << 4) + (k & 7) * 2;
}
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = static_cast<uint64_t>((saddr >> 4) & 0x3FFF);  // start address
  d |= static_cast<uint64_t>(1) << 16;                          // leading offset (unused with this swizzle)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;                  // 8-row groups 1024 B apart
  d |= static_cast<uint64_t>(1) << 46;                          // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                          // 128-byte swizzle
  return d;
}
// kind::f16 instruction descriptor: fp32 accumulate, fp16 A and B, both K-major, M = 128
__host__ __device__ constexpr uint32_t idesc_m128(uint32_t n) { return (1u << 4) | ((n >> 3) << 17) | ((128u >> 4) << 24); }

__device__ __forceinline__ void mma_f16(uint32_t dtmem, uint64_t da, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
          dtmem),
      "l"(da), "l"(db), "r"(idesc), "r"(acc));
}
// A from TMEM (one row per lane, fp16 pairs per 32-bit column), B from shared memory
__device__ __forceinline__ void mma_f16_ta(uint32_t dtmem, uint32_t atmem, uint64_t db, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(
          dtmem),
      "r"(atmem), "l"(db), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane
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
// 32 consecutive fp32 columns of this thread's TMEM lane from registers
__device__ __forceinline__ void tmem_st32(uint32_t addr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(addr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// 16 consecutive 32-bit columns of this thread's TMEM lane from registers
__device__ __forceinline__ void tmem_st16(uint32_t addr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          addr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]),
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ float tmem_ld1(uint32_t addr) {
  uint32_t r;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(addr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" : "+r"(r));
  return __uint_as_float(r);
}
__device__ __forceinline__ void fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// fp32 pair -> fp16 hi and fp16 lo with v = hi + lo * 2^-11 to about 2^-22
// relative.  The residual is carried scaled by 2^11 (|lo| <= |hi|) so that it
// stays a normal fp16 number whenever hi is: an unscaled residual of a value
// below 0.125 would be subnormal.  Products with hi and with lo accumulate in
// separate fp32 accumulators, combined as D_hi + D_lo * 2^-11.
constexpr float kLoScale = 2048.f, kLoInv = 1.f / 2048.f;
__device__ __forceinline__ uint32_t hi_lo2(float2 v, uint32_t& lo) {
  const __half2 hv = __float22half2_rn(v);
  const float2 hf = __half22float2(hv);
  const float2 r = __fadd2_rn(v, make_float2(-hf.x, -hf.y));
  lo = h2_as_u32(__float22half2_rn(__fmul2_rn(r, make_float2(kLoScale, kLoScale))));
  return h2_as_u32(hv);
}
__device__ __forceinline__ uint4 hi_lo_pack(const float (&x)[8], uint4& lo) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) h[k] = hi_lo2(make_float2(x[2 * k], x[2 * k + 1]), l[k]);
  lo = make_uint4(l[0], l[1], l[2], l[3]);
  return make_uint4(h[0], h[1], h[2], h[3]);
}
// 2^x for x <= 0 (the hardware approximation; -inf gives 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ------------------------------------------------------------------ kernel
// H (Sylvester, +-1) times the channel signs s_k as a K-major operand at
// `off`: element (r, k) = (-1)^popcount(r & k) s_k, or without signs.
__device__ void build_h(unsigned char* smem, int off, uint32_t seed) {
  for (int i = threadIdx.x; i < kHeadDim * 16; i += kPfThreads) {
    const int r = i >> 4, pc = i & 15;
    uint32_t w[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 8 * pc + 2 * k;
      const float x0 = ((__popc(r & c) & 1) ? -1.f : 1.f) * rotation_sign(seed, c);
      const float x1 = ((__popc(r & (c + 1)) & 1) ? -1.f : 1.f) * rotation_sign(seed, c + 1);
      w[k] = h2_as_u32(__floats2half2_rn(x0, x1));
    }
    *reinterpret_cast<uint4*>(smem + off + sw_off(r, 8 * pc, kHeadDim)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// query rows (raw fp16) of this CTA into the q''_hi area; rows past the chunk: zeros
__device__ void load_q_rows(unsigned char* smem, const PrefillArgs& a, int c0, int h, int rt, int rows_valid) {
  const int G = a.cfg.group_size, hqn = a.cfg.num_kv_heads * G;
  for (int i = threadIdx.x; i < kRows * 16; i += kPfThreads) {
    const int r = i >> 4, pc = i & 15;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < rows_valid) {
      const int gr = rt * kRows + r;
      v = *reinterpret_cast<const uint4*>(static_cast<const __half*>(a.q) +
                                          (static_cast<size_t>(c0 + gr / G) * hqn + h * G + gr % G) * kHeadDim +
                                          8 * pc);
    }
    *reinterpret_cast<uint4*>(smem + kOffAqHi + sw_off(r, 8 * pc, kRows)) = v;
  }
}

// one thread: D_hi = A_hi . B^T (and D_lo = A_lo . B^T when npass = 2, A_lo
// `a_lo` bytes after A_hi) over K = 16 * ksteps; atoms of A 16 KB apart, of B
// `b_atom` apart
__device__ __forceinline__ void issue_mma(uint32_t d_hi, uint32_t d_lo, uint32_t a0, uint32_t a_lo, int npass,
                                          uint32_t b0, uint32_t b_atom, int ksteps, uint32_t idesc, uint32_t bar) {
  fence_after();
  for (int hl = 0; hl < npass; ++hl) {
    const uint32_t sa = a0 + hl * a_lo;
    for (int s = 0; s < ksteps; ++s) {
      const uint32_t ka = (s >> 2) * 16384 + (s & 3) * 32, kb = (s >> 2) * b_atom + (s & 3) * 32;
      mma_f16(hl ? d_lo : d_hi, sw128_desc(sa + ka), sw128_desc(b0 + kb), idesc, s != 0);
    }
  }
  mma_commit(bar);
}

// one thread: D_hi = q''_hi . B_K^T and D_lo = q''_lo . B_K^T with q'' in
// TMEM (hi at column a_hi, lo 64 columns on; 8 columns per 16-element K step)
__device__ __forceinline__ void issue_qk_ta(uint32_t d_hi, uint32_t d_lo, uint32_t a_hi, uint32_t b0, uint32_t bar) {
  fence_after();
#pragma unroll
  for (int hl = 0; hl < 2; ++hl)
#pragma unroll
    for (int s = 0; s < 8; ++s)
      mma_f16_ta(hl ? d_lo : d_hi, a_hi + 64 * hl + 8 * s, sw128_desc(b0 + (s >> 2) * kBkAtom + (s & 3) * 32),
                 idesc_m128(kNS), s != 0);
  mma_commit(bar);
}

__device__ __forceinline__ float f4_at(const float4& v, int k) {
  return k == 0 ? v.x : (k == 1 ? v.y : (k == 2 ? v.z : v.w));
}

template <int T, int BK, int BV>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_attn_kernel(PrefillArgs a) {
  using Geo = PfGeom<T, BK, BV>;
  constexpr int NP = Geo::kPages;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int quad = warp & 3, eta = warp >> 2;  // TMEM lane quadrant, column half
  const int row = 32 * quad + lane;            // this thread's query row (TMEM lane)
  const int G = a.cfg.group_size, nh = a.cfg.num_kv_heads;
  const int R = a.row_tiles;
  // mode 1: CTA = (unit, split of the context tiles); modes 0 and 2: CTA = unit
  const int S = a.mode == 1 ? a.num_splits : 1;
  const int unit = blockIdx.x / S, split = blockIdx.x % S;
  const int rt = unit % R, bh = unit / R;
  const int h = bh % nh, b = bh / nh;
  const int c0 = a.cu_chunk[b];
  const int n = a.cu_chunk[b + 1] - c0;
  if ((n < 0 || n > a.max_chunk) && tid == 0 && rt == 0 && h == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
  const int nc = max(0, min(n, a.max_chunk));  // chunk tokens served
  const int rows_valid = min(nc * G - rt * kRows, kRows);
  if (rows_valid <= 0) return;
  const int L = max(a.ctx_lens[b], 0);
  const int F = L / T, tau = L - F * T;
  // the context tiles this CTA runs through: all (mode 0), its split's share
  // (mode 1), none (mode 2: it combines the splits' partials instead)
  const int t_lo = a.mode == 1 ? static_cast<int>(static_cast<long long>(F) * split / S) : 0;
  const int t_hi = a.mode == 1 ? static_cast<int>(static_cast<long long>(F) * (split + 1) / S) : (a.mode == 0 ? F : 0);
  const int Fr = t_hi - t_lo;
  // chunk token of this thread's row (rows past the chunk take the last one)
  const int i_row = (rt * kRows + min(row, rows_valid - 1)) / G;
  const int i_max = (rt * kRows + rows_valid - 1) / G;
  if (a.mode == 1 && Fr == 0) {  // no context tile in this split: an empty partial, and no set-up at all
    if (row < rows_valid) {
      float* part = a.partials + (static_cast<size_t>(blockIdx.x) * kRows + row) * (4 + kHeadDim);
      if (eta == 0) *reinterpret_cast<float2*>(part) = make_float2(-INFINITY, 0.f);
#pragma unroll
      for (int i = 0; i < 64; i += 4) *reinterpret_cast<float4*>(part + 4 + 64 * eta + i) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }

  const uint32_t s_base = smem_u32(smem);
  const uint32_t bar_stage0 = s_base + kOffBar, bar_mma = s_base + kOffBar + 16;
  const uint32_t bar_qk = s_base + kOffBar + 24, bar_pv = s_base + kOffBar + 32;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  int* stage_bad = reinterpret_cast<int*>(smem + kOffMisc + 8);  // [2]
  float* red = reinterpret_cast<float*>(smem + kOffRed);          // [3][2][128]
  float* fbase = reinterpret_cast<float*>(smem + kOffF);          // tile scalars, buffer = tile parity
  int* tile_bad = reinterpret_cast<int*>(smem + kOffMisc + 16);   // [2], by tile parity
  const uint8_t* kpool = static_cast<const uint8_t*>(a.k_pool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.v_pool);

  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_stage0));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_stage0 + 8));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_mma));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_qk));
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar_pv));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)), "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }

  // warp 0 stages tile `tile` (all K pages, then all V pages) into stage st;
  // bit st of `issued` (warp 0's copy) marks copies not yet waited for
  uint32_t issued = 0u;
  auto issue = [&](int tile, int st) {
    const int lb = tile * NP + lane;
    int blk = -1;
    if (lane < NP)
      blk = lb < a.max_blocks_per_seq ? a.block_tables[static_cast<size_t>(b) * a.max_blocks_per_seq + lb] : -1;
    const bool bad = lane < NP && (blk < 0 || blk >= a.num_blocks);
    if (__any_sync(kFull, bad)) {
      if (lane == 0) {
        report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
        stage_bad[st] = 1;
      }
      return;
    }
    if (lane == 0) {
      stage_bad[st] = 0;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar_stage0 + 8 * st),
                   "r"(NP * (Geo::kPageK + Geo::kPageV))
                   : "memory");
    }
    __syncwarp();
    if (lane < NP) {
      const uint32_t dst = s_base + kOffStage + st * Geo::kStage;
      const size_t reg = static_cast<size_t>(blk) * nh + h;
      bulk_g2s(dst + lane * Geo::kPageK, kpool + reg * Geo::kPageK, Geo::kPageK, bar_stage0 + 8 * st);
      bulk_g2s(dst + NP * Geo::kPageK + lane * Geo::kPageV, vpool + reg * Geo::kPageV, Geo::kPageV,
               bar_stage0 + 8 * st);
    }
    issued |= 1u << st;
  };
  __syncthreads();  // barriers initialised
  if (warp == 0 && Fr > 0) issue(t_lo, 0);

  const uint32_t t_lane = static_cast<uint32_t>(32 * quad) << 16;
  uint32_t tbase = 0, mma_phase = 0;
  bool ok = true;
  float acc[64];  // rotated-domain accumulator of the context
#pragma unroll
  for (int i = 0; i < 64; ++i) acc[i] = 0.f;
  float m_ctx = -INFINITY, l_ctx = 0.f;

  // ---- set-up: q rows and H D_s; q' = q D_s H on the tensor cores
  load_q_rows(smem, a, c0, h, rt, rows_valid);
  build_h(smem, kOffBk, a.cfg.rotation_seed);
  fence_async_smem();
  fence_before();
  __syncthreads();
  fence_after();
  tbase = *tslot;
  // TMEM columns: D_S 0..79, D_O 128..255, 256..383 q' (context part), then
  // the parked context accumulator (raw part); 384..447 / 448..511 q''_hi /
  // q''_lo as the QK MMA's A operand (row = lane, 2 fp16 per column).  The lo
  // products of QK go to 128..207 (D_O is free then), those of PV to 0..127
  // (D_S is free then).
  const uint32_t d_s = tbase, d_o = tbase + 128, d_park = tbase + 256, a_q = tbase + 384;
  if (Fr > 0) {
    if (tid == 0)
      issue_mma(d_o, d_o, s_base + kOffAqHi, 0, 1, s_base + kOffBk, 16384, 8, idesc_m128(kHeadDim), bar_mma);
    ok = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1u;
    fence_after();
    const float qscale = a.softmax_scale * kLog2e / kSqrtHeadDim;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float x[32];
      tmem_ld32(d_o + t_lane + 64 * eta + 32 * half, x);
#pragma unroll
      for (int i = 0; i < 32; ++i) x[i] *= qscale;
      tmem_st32(d_park + t_lane + 64 * eta + 32 * half, x);
    }
    fence_before();
  }
  __syncthreads();
  // B_K, B_V, P start zeroed (padding rows / tokens stay zero); B_K row 64 = ones
  for (int i = tid; i < (kOffRed - kOffBk) / 16; i += kPfThreads)
    *reinterpret_cast<uint4*>(smem + kOffBk + 16 * i) = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (tid < 16)
    *reinterpret_cast<uint4*>(smem + kOffBk + sw_off(kBlk, 8 * tid, kNS)) =
        make_uint4(0x3C003C00u, 0x3C003C00u, 0x3C003C00u, 0x3C003C00u);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
    ok = false;
  }

  // ================================================================ A. context tiles
  // Loop over the context's 64-token blocks gb = 0 .. NB-1.  Block gb+1's
  // codes (and, on a tile change, the next tile's scalars) are unpacked in
  // shared memory while PV(gb) runs; the TMEM reads of the accumulator fold
  // and the next tile's q'' build wait until no MMA is in flight (an MMA
  // writing TMEM slows concurrent tcgen05.ld), then QK(gb+1) is issued.
  const int NB = Fr * Geo::kBlocks;  // tile indices below are relative to t_lo
  uint32_t st_phase = 0u, qk_phase = 0u, pv_phase = 0u;  // st_phase bit s: stage s

  // tile t, shared memory only: wait for its pages (skipped when outside the
  // pool: the tile's blocks then run with zero scalars and masked scores),
  // stage the tile scalars as floats; starts the copies of tile t+1.  Has no
  // barrier of its own: returns this thread's wait result, which the caller
  // folds into its next barrier (that barrier also publishes the scalars).
  auto prep_scalars = [&](int t) -> bool {
    const int st = t & 1;
    if (warp == 0 && t + 1 < Fr) issue(t_lo + t + 1, st ^ 1);
    const bool bad = stage_bad[st] != 0;
    bool got = true;
    if (!bad) {
      got = mbar_wait(bar_stage0 + 8 * st, (st_phase >> st) & 1u);
      st_phase ^= 1u << st;
      if (got) issued &= ~(1u << st);
    }
    const unsigned char* sK = smem + kOffStage + st * Geo::kStage;
    const unsigned char* sV = sK + NP * Geo::kPageK;
    float* f = fbase + st * kFBuf;
    if (tid < kHeadDim) {
      const int c = tid, pg = c / Geo::kCs, o = 2 * (c % Geo::kCs);
      f[c] = bad ? 0.f : __half2float(*reinterpret_cast<const __half*>(sK + pg * Geo::kPageK + Geo::kCodesK + 64 + o));
      f[128 + c] =
          bad ? 0.f : __half2float(*reinterpret_cast<const __half*>(sV + pg * Geo::kPageV + Geo::kCodesV + 64 + o));
    } else if (tid - kHeadDim < T) {
      const int tok = tid - kHeadDim, pg = tok / kPageTokens, o = 4 * (tok % kPageTokens);
      float2 k2 = make_float2(0.f, 0.f), v2 = make_float2(0.f, 0.f);
      if (!bad) {
        k2 = __half22float2(*reinterpret_cast<const __half2*>(sK + pg * Geo::kPageK + Geo::kCodesK + o));
        v2 = __half22float2(*reinterpret_cast<const __half2*>(sV + pg * Geo::kPageV + Geo::kCodesV + o));
      }
      f[256 + tok] = k2.x;
      f[384 + tok] = k2.y;
      f[512 + tok] = v2.x;
      f[640 + tok] = v2.y;
    }
    if (tid == 0) tile_bad[st] = bad;
    return got;
  };
  // tile t's q'' = q' * C~K (hi / lo) into TMEM in the QK channel order; the
  // scalars of tile t must be visible (a barrier after prep_scalars)
  auto build_qpp = [&](int t) {
    const float* f = fbase + (t & 1) * kFBuf;
    // q'' pieces 4 half .. 4 half + 3 use channels 32 half .. 32 half + 31 of
    // this thread's 64 (a word's channel group never straddles 32); MMA
    // positions 64 eta + 32 half .. +31 go to 16 TMEM columns each for hi, lo
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float qv[32];
      tmem_ld32(d_park + t_lane + 64 * eta + 32 * half, qv);
      uint32_t whi[16], wlo[16];
#pragma unroll
      for (int pq = 0; pq < 4; ++pq) {
        const int pc = 4 * half + pq;
        constexpr int kSecond = BK == 2 ? 8 : 4;  // the piece's channels: two aligned groups of 4
        const int first = qk_channel<BK>(8 * pc);
        const float4 g0 = *reinterpret_cast<const float4*>(f + 64 * eta + first);
        const float4 g1 = *reinterpret_cast<const float4*>(f + 64 * eta + first + kSecond);
        float x[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const int cl = qk_channel<BK>(8 * pc + m);
          const float cval = cl < first + 4 ? f4_at(g0, cl - first) : f4_at(g1, cl - first - kSecond);
          x[m] = qv[cl - 32 * half] * cval;
        }
        uint4 lo;
        const uint4 hi = hi_lo_pack(x, lo);
        whi[4 * pq] = hi.x;
        whi[4 * pq + 1] = hi.y;
        whi[4 * pq + 2] = hi.z;
        whi[4 * pq + 3] = hi.w;
        wlo[4 * pq] = lo.x;
        wlo[4 * pq + 1] = lo.y;
        wlo[4 * pq + 2] = lo.z;
        wlo[4 * pq + 3] = lo.w;
      }
      tmem_st16(a_q + t_lane + 32 * eta + 16 * half, whi);
      tmem_st16(a_q + 64 + t_lane + 32 * eta + 16 * half, wlo);
    }
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
  };

  // block gb's codes: K into B_K (token rows), V into B_V buffer gb & 1
  // (channel rows, token pairs; lane L = 4 g + t of a page owns words k in
  // 16-byte rows k / 4, word k holding channels 8 (h (k / 2) + e) + g for
  // tokens 2t + 8 (k % 2) and the next, h = 16 / b pairs per word)
  auto unpack_block = [&](int gb) {
    const int t = gb / Geo::kBlocks, kb = gb % Geo::kBlocks;
    const unsigned char* sK = smem + kOffStage + (t & 1) * Geo::kStage;
    const unsigned char* sV = sK + NP * Geo::kPageK;
    const int pg0 = kb * (kBlk / kPageTokens);
    for (int i = tid; i < Geo::kValid * 16; i += kPfThreads) {
      const int tok = i >> 4, pc = i & 15;
      const unsigned char* rec = sK + (pg0 + tok / kPageTokens) * Geo::kPageK + (tok % kPageTokens) * (16 * BK);
      uint32_t pr[4];
      if constexpr (BK == 3) {  // channels 8 pc .. 8 pc + 7: bits 24 pc .. 24 pc + 23 of the record
        const uint32_t* rw = reinterpret_cast<const uint32_t*>(rec);
        const uint32_t x = field_at<24>(rw, 24 * pc);
#pragma unroll
        for (int k = 0; k < 4; ++k) pr[k] = code_pair_f16((x >> (6 * k)) & 7u, (x >> (6 * k + 3)) & 7u);
      } else if constexpr (BK == 4) {
        unpack_pairs<4>(*reinterpret_cast<const uint32_t*>(rec + 4 * pc), pr);
      } else if constexpr (BK == 2) {
        uint32_t all[8];
        unpack_pairs<2>(*reinterpret_cast<const uint32_t*>(rec + 4 * (pc >> 1)), all);
#pragma unroll
        for (int k = 0; k < 4; ++k) pr[k] = (pc & 1) ? all[4 + k] : all[k];
      } else {
        const uint2 w = *reinterpret_cast<const uint2*>(rec + 8 * pc);
        unpack_pairs<8>(w.x, pr);
        unpack_pairs<8>(w.y, pr + 2);
      }
      *reinterpret_cast<uint4*>(smem + kOffBk + sw_off(tok, 8 * pc, kNS)) = make_uint4(pr[0], pr[1], pr[2], pr[3]);
    }
    unsigned char* bv = smem + kOffBv + (gb & 1) * 16384;
    if constexpr (BV == 3) {
      // 3-bit V pages are a token-major bitstream: code (token p, channel c)
      // at bit 3 (128 p + c); each unit is one channel of one token pair
      constexpr int kUnits3 = (Geo::kValid / kPageTokens) * kHeadDim * (kPageTokens / 2);
      for (int i = tid; i < kUnits3; i += kPfThreads) {
        const int pgl = i / (kHeadDim * (kPageTokens / 2)), rem = i % (kHeadDim * (kPageTokens / 2));
        const int c = rem % kHeadDim, j = rem / kHeadDim;
        const uint32_t* cw = reinterpret_cast<const uint32_t*>(sV + (pg0 + pgl) * Geo::kPageV);
        const int bit = 3 * (kHeadDim * 2 * j + c);
        *reinterpret_cast<uint32_t*>(bv + sw_off(c, kPageTokens * pgl + 2 * j, kHeadDim)) =
            code_pair_f16(field_at<3>(cw, bit), field_at<3>(cw, bit + 3 * kHeadDim));
      }
      return;
    }
    constexpr int kRowsPerLane = BV / 2;  // 16-byte rows per lane (2 b words / 4)
    constexpr int kVUnits = (Geo::kValid / kPageTokens) * 32 * kRowsPerLane;
    for (int i = tid; i < kVUnits; i += kPfThreads) {
      const int pgl = i / (32 * kRowsPerLane), rem = i % (32 * kRowsPerLane);
      const int j = rem / 32, ln = rem % 32;
      const uint4 v4 = *reinterpret_cast<const uint4*>(sV + (pg0 + pgl) * Geo::kPageV + (j * 32 + ln) * 16);
      const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
      const int g8 = ln >> 2, tt = ln & 3;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = 4 * j + q;
        constexpr int hV = 16 / BV;
        uint32_t pr[hV];
        unpack_pairs<BV>(wv[q], pr);
        const int kpos = kPageTokens * pgl + 2 * tt + 8 * (k & 1);
#pragma unroll
        for (int e = 0; e < hV; ++e) {
          const int c = 8 * (hV * (k >> 1) + e) + g8;
          *reinterpret_cast<uint32_t*>(bv + sw_off(c, kpos, kHeadDim)) = pr[e];
        }
      }
    }
  };

  if (NB > 0 && ok) {
    const bool got0 = prep_scalars(0);
    unpack_block(0);
    if (__syncthreads_or(!got0)) {  // scalars of tile 0 visible
      if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
      ok = false;
    }
    if (ok) {
      build_qpp(0);
      fence_async_smem();
      fence_before();
      __syncthreads();
      if (tid == 0) issue_qk_ta(d_s, d_o, a_q, s_base + kOffBk, bar_qk);
    }
  }
  for (int gb = 0; gb < NB && ok; ++gb) {
    const int t = gb / Geo::kBlocks, kb = gb % Geo::kBlocks;
    const float* f = fbase + (t & 1) * kFBuf;
    // -- scores of block gb (log2 domain) once QK(gb) is done, block max
    const bool got_s = mbar_wait(bar_qk, qk_phase);
    qk_phase ^= 1u;
    fence_after();
    const bool live = 32 * eta < Geo::kValid;  // warp-uniform
    const bool masked = tile_bad[t & 1] != 0;  // block-uniform
    const int tok0 = kBlk * kb + 32 * eta;     // first token (within the tile) of this thread
    float sc[32];
    float mloc = -INFINITY;
    if (live) {
      {
        float lo[32];
        tmem_ld32(d_s + t_lane + 32 * eta, sc);
        tmem_ld32(d_o + t_lane + 32 * eta, lo);
#pragma unroll
        for (int j = 0; j < 32; j += 2) {
          const float2 v = __ffma2_rn(make_float2(lo[j], lo[j + 1]), make_float2(kLoInv, kLoInv),
                                      make_float2(sc[j], sc[j + 1]));
          sc[j] = v.x;
          sc[j + 1] = v.y;
        }
      }
      const float sig = tmem_ld1(d_s + t_lane + kBlk) + tmem_ld1(d_o + t_lane + kBlk) * kLoInv;
      const float2 sig2 = make_float2(sig, sig);
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const float4 s4 = *reinterpret_cast<const float4*>(f + 256 + tok0 + 4 * j4);
        const float4 z4 = *reinterpret_cast<const float4*>(f + 384 + tok0 + 4 * j4);
        const float2 v0 = __ffma2_rn(make_float2(s4.x, s4.y), make_float2(sc[4 * j4], sc[4 * j4 + 1]),
                                     __fmul2_rn(make_float2(z4.x, z4.y), sig2));
        const float2 v1 = __ffma2_rn(make_float2(s4.z, s4.w), make_float2(sc[4 * j4 + 2], sc[4 * j4 + 3]),
                                     __fmul2_rn(make_float2(z4.z, z4.w), sig2));
        sc[4 * j4] = v0.x;
        sc[4 * j4 + 1] = v0.y;
        sc[4 * j4 + 2] = v1.x;
        sc[4 * j4 + 3] = v1.y;
        mloc = fmaxf(mloc, fmaxf(fmaxf(v0.x, v0.y), fmaxf(v1.x, v1.y)));
      }
      if (masked) {
#pragma unroll
        for (int j = 0; j < 32; ++j) sc[j] = -INFINITY;
        mloc = -INFINITY;
      }
    }
    red[eta * kRows + row] = mloc;
    if (__syncthreads_or(!got_s)) {
      if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
      ok = false;
      break;
    }
    const float m_new = fmaxf(m_ctx, fmaxf(red[row], red[kRows + row]));
    const bool none = m_new == -INFINITY;  // nothing seen yet (masked blocks only)
    const float alpha = none ? 1.f : ex2(m_ctx - m_new);
    const float m_use = none ? 0.f : m_new;  // p = 2^(-inf) = 0 either way
    // -- P = p * s~V (hi / lo), sums of p and p z~V (PV(gb-1) is done: its P is free)
    float2 lsum2 = make_float2(0.f, 0.f), wsum2 = make_float2(0.f, 0.f);
    if (live) {
      const float2 mneg = make_float2(-m_use, -m_use);
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t h[4], l[4];
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const float4 s4 = *reinterpret_cast<const float4*>(f + 512 + tok0 + 8 * pc + 4 * hf);
          const float4 z4 = *reinterpret_cast<const float4*>(f + 640 + tok0 + 8 * pc + 4 * hf);
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const int j = 8 * pc + 4 * hf + 2 * k2;
            const float2 e = __fadd2_rn(make_float2(sc[j], sc[j + 1]), mneg);
            const float2 p2 = make_float2(ex2(e.x), ex2(e.y));
            const float2 sv = k2 ? make_float2(s4.z, s4.w) : make_float2(s4.x, s4.y);
            const float2 zv = k2 ? make_float2(z4.z, z4.w) : make_float2(z4.x, z4.y);
            lsum2 = __fadd2_rn(lsum2, p2);
            wsum2 = __ffma2_rn(p2, zv, wsum2);
            h[2 * hf + k2] = hi_lo2(__fmul2_rn(p2, sv), l[2 * hf + k2]);
          }
        }
        const int kpos = 32 * eta + 8 * pc;
        *reinterpret_cast<uint4*>(smem + kOffPHi + sw_off(row, kpos, kRows)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(smem + kOffPLo + sw_off(row, kpos, kRows)) = make_uint4(l[0], l[1], l[2], l[3]);
      }
    }
    red[(1 * 2 + eta) * kRows + row] = lsum2.x + lsum2.y;
    red[(2 * 2 + eta) * kRows + row] = wsum2.x + wsum2.y;
    fence_async_smem();
    fence_before();
    __syncthreads();
    if (tid == 0)
      issue_mma(d_o, d_s, s_base + kOffPHi, kOffPLo - kOffPHi, 2, s_base + kOffBv + (gb & 1) * 16384, 16384, 4,
                idesc_m128(kHeadDim), bar_pv);
    l_ctx = l_ctx * alpha + red[2 * kRows + row] + red[3 * kRows + row];
    const float wtot = red[4 * kRows + row] + red[5 * kRows + row];
    m_ctx = m_new;
    // -- while PV(gb) runs (shared memory only): block gb+1's codes and, on a
    // tile change, the next tile's scalars
    const bool more = gb + 1 < NB;
    const bool new_tile = more && (gb + 1) % Geo::kBlocks == 0;
    const bool got_t = new_tile ? prep_scalars((gb + 1) / Geo::kBlocks) : true;
    if (more) unpack_block(gb + 1);  // (garbage after a timed-out wait; dropped below)
    // -- fold D_O into the accumulators: acc'_c = alpha acc'_c + C~V_c (D_c + sum p z~V)
    const bool got_o = mbar_wait(bar_pv, pv_phase);
    pv_phase ^= 1u;
    fence_after();
    const float2 alpha2 = make_float2(alpha, alpha), w2 = make_float2(wtot, wtot);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float x[32];
      {
        float lo[32];
        tmem_ld32(d_o + t_lane + 64 * eta + 32 * half, x);
        tmem_ld32(d_s + t_lane + 64 * eta + 32 * half, lo);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 v = __ffma2_rn(make_float2(lo[i], lo[i + 1]), make_float2(kLoInv, kLoInv),
                                      make_float2(x[i], x[i + 1]));
          x[i] = v.x;
          x[i + 1] = v.y;
        }
      }
#pragma unroll
      for (int i4 = 0; i4 < 8; ++i4) {
        const float4 c4 = *reinterpret_cast<const float4*>(f + 128 + 64 * eta + 32 * half + 4 * i4);
#pragma unroll
        for (int k2 = 0; k2 < 2; ++k2) {
          const int i = 32 * half + 4 * i4 + 2 * k2;
          const float2 cv = k2 ? make_float2(c4.z, c4.w) : make_float2(c4.x, c4.y);
          const float2 r = __ffma2_rn(alpha2, make_float2(acc[i], acc[i + 1]),
                                      __fmul2_rn(cv, __fadd2_rn(make_float2(x[4 * i4 + 2 * k2], x[4 * i4 + 2 * k2 + 1]), w2)));
          acc[i] = r.x;
          acc[i + 1] = r.y;
        }
      }
    }
    // -- no MMA in flight: the next tile's q'' into TMEM, then QK(gb+1)
    if (new_tile) {
      fence_before();
      if (__syncthreads_or(!got_t)) {  // next tile's scalars visible; D_O reads done
        if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
        ok = false;
      }
      fence_after();
      if (ok) build_qpp((gb + 1) / Geo::kBlocks);
    }
    fence_async_smem();
    fence_before();
    if (__syncthreads_or(!got_o)) {
      if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
      ok = false;
    }
    if (more && ok && tid == 0) issue_qk_ta(d_s, d_o, a_q, s_base + kOffBk, bar_qk);
  }

  if (a.mode == 1) {  // split partial: (m, l, acc') of this row over the split's tiles
    if (row < rows_valid) {
      float* part = a.partials + (static_cast<size_t>(blockIdx.x) * kRows + row) * (4 + kHeadDim);
      if (eta == 0) *reinterpret_cast<float2*>(part) = make_float2(m_ctx, l_ctx);
#pragma unroll
      for (int i = 0; i < 64; i += 4)
        *reinterpret_cast<float4*>(part + 4 + 64 * eta + i) = make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]);
    }
    if (!ok && warp == 0) {  // let copies in flight land before the shared memory is released
      for (int s = 0; s < 2; ++s)
        if (issued & (1u << s)) (void)mbar_wait(bar_stage0 + 8 * s, (st_phase >> s) & 1u);
    }
    fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(512));
    return;
  }
  if (a.mode == 2 && F > 0 && row < rows_valid) {  // combine the splits' partials (log-sum-exp)
    const float* part0 = a.partials + (static_cast<size_t>(unit) * a.num_splits * kRows + row) * (4 + kHeadDim);
    const size_t sstride = static_cast<size_t>(kRows) * (4 + kHeadDim);
    for (int sp = 0; sp < a.num_splits; ++sp) {
      const float2 ml = *reinterpret_cast<const float2*>(part0 + sp * sstride);
      if (ml.y > 0.f) m_ctx = fmaxf(m_ctx, ml.x);
    }
    for (int sp = 0; sp < a.num_splits; ++sp) {
      const float* pp = part0 + sp * sstride;
      const float2 ml = *reinterpret_cast<const float2*>(pp);
      if (!(ml.y > 0.f)) continue;
      const float wgt = ex2(ml.x - m_ctx);
      l_ctx += wgt * ml.y;
#pragma unroll
      for (int i = 0; i < 64; i += 4) {
        const float4 v = *reinterpret_cast<const float4*>(pp + 4 + 64 * eta + i);
        acc[i] += wgt * v.x;
        acc[i + 1] += wgt * v.y;
        acc[i + 2] += wgt * v.z;
        acc[i + 3] += wgt * v.w;
      }
    }
  }

  // ================================================================ B. raw keys
  // keys j: the tail (j < tau), then chunk rows j - tau; row i sees j <= tau + i.
  // The context accumulator waits in TMEM meanwhile.
  if (F > 0) {
    float x[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = acc[i];
    tmem_st32(d_park + t_lane + 64 * eta, x);
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = acc[32 + i];
    tmem_st32(d_park + t_lane + 64 * eta + 32, x);
  }
  float m_raw = -INFINITY, l_raw = 0.f;
  float racc[64];  // the raw-part accumulator (original domain)
#pragma unroll
  for (int i = 0; i < 64; ++i) racc[i] = 0.f;
  const int nkeys = tau + i_max + 1;
  if (ok) load_q_rows(smem, a, c0, h, rt, rows_valid);
  const float rscale = a.softmax_scale * kLog2e;
  const __half* kt = static_cast<const __half*>(a.k_tail) + (static_cast<size_t>(b) * nh + h) * T * kHeadDim;
  const __half* vt = static_cast<const __half*>(a.v_tail) + (static_cast<size_t>(b) * nh + h) * T * kHeadDim;
  const __half* kn = static_cast<const __half*>(a.k_new) + (static_cast<size_t>(c0) * nh + h) * kHeadDim;
  const __half* vn = static_cast<const __half*>(a.v_new) + (static_cast<size_t>(c0) * nh + h) * kHeadDim;
  const size_t new_stride = static_cast<size_t>(nh) * kHeadDim;
  auto key_row = [&](int j, bool val) -> const __half* {
    if (j < tau) return (val ? vt : kt) + static_cast<size_t>(j) * kHeadDim;
    return (val ? vn : kn) + static_cast<size_t>(j - tau) * new_stride;
  };
  for (int j0 = 0; j0 < nkeys && ok; j0 += kBlk) {
    // -- K rows into B_K (keys past the end: zeros), V rows transposed into B_V
    for (int i = tid; i < kBlk * 16; i += kPfThreads) {
      const int r = i >> 4, pc = i & 15;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (j0 + r < nkeys) v = *reinterpret_cast<const uint4*>(key_row(j0 + r, false) + 8 * pc);
      *reinterpret_cast<uint4*>(smem + kOffBk + sw_off(r, 8 * pc, kNS)) = v;
    }
    for (int i = tid; i < (kBlk / 2) * 16; i += kPfThreads) {
      const int r2 = i >> 4, pc = i & 15;  // keys 2 r2, 2 r2 + 1; channels 8 pc ..
      uint4 v0 = make_uint4(0, 0, 0, 0), v1 = make_uint4(0, 0, 0, 0);
      if (j0 + 2 * r2 < nkeys) v0 = *reinterpret_cast<const uint4*>(key_row(j0 + 2 * r2, true) + 8 * pc);
      if (j0 + 2 * r2 + 1 < nkeys) v1 = *reinterpret_cast<const uint4*>(key_row(j0 + 2 * r2 + 1, true) + 8 * pc);
      const uint32_t a4[4] = {v0.x, v0.y, v0.z, v0.w}, b4[4] = {v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        // channels 8 pc + 2k (low halves) and 8 pc + 2k + 1 (high halves)
        *reinterpret_cast<uint32_t*>(smem + kOffBv + sw_off(8 * pc + 2 * k, 2 * r2, kHeadDim)) =
            __byte_perm(a4[k], b4[k], 0x5410);
        *reinterpret_cast<uint32_t*>(smem + kOffBv + sw_off(8 * pc + 2 * k + 1, 2 * r2, kHeadDim)) =
            __byte_perm(a4[k], b4[k], 0x7632);
      }
    }
    fence_async_smem();
    __syncthreads();
    if (tid == 0)
      issue_mma(d_s, d_s, s_base + kOffAqHi, 0, 1, s_base + kOffBk, kBkAtom, 8, idesc_m128(kBlk), bar_mma);
    const bool got_s = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1u;
    fence_after();
    float sc[32];
    float mloc = -INFINITY;
    const int jt = j0 + 32 * eta;  // first key of this thread
    const bool live = jt < nkeys;  // warp-uniform
    if (live) {
      tmem_ld32(d_s + t_lane + 32 * eta, sc);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        sc[j] = (jt + j <= tau + i_row) ? sc[j] * rscale : -INFINITY;
        mloc = fmaxf(mloc, sc[j]);
      }
    }
    red[eta * kRows + row] = mloc;
    if (__syncthreads_or(!got_s)) {
      if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
      ok = false;
      break;
    }
    const float m_new = fmaxf(m_raw, fmaxf(red[row], red[kRows + row]));
    const float alpha = ex2(m_raw - m_new);
    float lsum = 0.f;
    if (live) {
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        float x[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float p = ex2(sc[8 * pc + m] - m_new);
          lsum += p;
          x[m] = p;
        }
        uint4 lo;
        const uint4 hi = hi_lo_pack(x, lo);
        const int kpos = 32 * eta + 8 * pc;
        *reinterpret_cast<uint4*>(smem + kOffPHi + sw_off(row, kpos, kRows)) = hi;
        *reinterpret_cast<uint4*>(smem + kOffPLo + sw_off(row, kpos, kRows)) = lo;
      }
    } else {  // keys past the end: P stays zero for them
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        const int kpos = 32 * eta + 8 * pc;
        *reinterpret_cast<uint4*>(smem + kOffPHi + sw_off(row, kpos, kRows)) = make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(smem + kOffPLo + sw_off(row, kpos, kRows)) = make_uint4(0, 0, 0, 0);
      }
    }
    red[(2 + eta) * kRows + row] = lsum;
    fence_async_smem();
    fence_before();
    __syncthreads();
    if (tid == 0)
      issue_mma(d_o, d_s, s_base + kOffPHi, kOffPLo - kOffPHi, 2, s_base + kOffBv, 16384, 4, idesc_m128(kHeadDim),
                bar_mma);
    l_raw = l_raw * alpha + red[2 * kRows + row] + red[3 * kRows + row];
    m_raw = m_new;
    const bool got_o = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1u;
    fence_after();
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float x[32], lo[32];
      tmem_ld32(d_o + t_lane + 64 * eta + 32 * half, x);
      tmem_ld32(d_s + t_lane + 64 * eta + 32 * half, lo);
#pragma unroll
      for (int i = 0; i < 32; ++i) racc[32 * half + i] = alpha * racc[32 * half + i] + (x[i] + lo[i] * kLoInv);
    }
    fence_before();
    if (__syncthreads_or(!got_o)) {
      if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
      ok = false;
    }
  }

  // ================================================================ C. merge, inverse rotation, output
  const float m_all = fmaxf(m_ctx, m_raw);
  const float w_ctx = l_ctx > 0.f ? exp2f(m_ctx - m_all) : 0.f;
  const float w_raw = l_raw > 0.f ? exp2f(m_raw - m_all) : 0.f;
  const float inv_l = 1.f / (l_ctx * w_ctx + l_raw * w_raw);
  bool have_rot = F > 0 && ok;  // block-uniform
  if (have_rot) {
    // acc' (times its weight) in hi / lo halves as the A operand, H (no signs) as B
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float y[32];
      tmem_ld32(d_park + t_lane + 64 * eta + 32 * half, y);
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        float x[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) x[m] = y[8 * pc + m] * (w_ctx * inv_l);  // bounded by max |V|
        uint4 lo;
        const uint4 hi = hi_lo_pack(x, lo);
        const int kpos = 64 * eta + 32 * half + 8 * pc;
        *reinterpret_cast<uint4*>(smem + kOffAqHi + sw_off(row, kpos, kRows)) = hi;
        *reinterpret_cast<uint4*>(smem + kOffAqLo + sw_off(row, kpos, kRows)) = lo;
      }
    }
    build_h(smem, kOffBv, 0u);
    fence_async_smem();
    __syncthreads();
    if (tid == 0)
      issue_mma(d_o, d_s, s_base + kOffAqHi, kOffAqLo - kOffAqHi, 2, s_base + kOffBv, 16384, 8, idesc_m128(kHeadDim),
                bar_mma);
    const bool got = mbar_wait(bar_mma, mma_phase);
    mma_phase ^= 1u;
    fence_after();
    if (__syncthreads_or(!got)) {
      if (tid == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
      ok = have_rot = false;
    }
  }
  {
    const int gr = rt * kRows + min(row, rows_valid - 1);
    __half* o = static_cast<__half*>(a.out) + (static_cast<size_t>(c0 + gr / G) * nh * G + h * G + gr % G) * kHeadDim +
                64 * eta;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      float x[32];
      if (have_rot) {
        float lo[32];
        tmem_ld32(d_o + t_lane + 64 * eta + 32 * half, x);
        tmem_ld32(d_s + t_lane + 64 * eta + 32 * half, lo);
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] += lo[i] * kLoInv;
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) x[i] = 0.f;
      }
#pragma unroll
      for (int pc = 0; pc < 4; ++pc) {
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int i = 8 * pc + 2 * k, c = 64 * eta + 32 * half + i;
          const float r0 = x[i] * (rotation_sign(a.cfg.rotation_seed, c) / kSqrtHeadDim);
          const float r1 = x[i + 1] * (rotation_sign(a.cfg.rotation_seed, c + 1) / kSqrtHeadDim);
          w[k] = h2_as_u32(__floats2half2_rn(r0 + racc[32 * half + i] * (w_raw * inv_l),
                                             r1 + racc[32 * half + i + 1] * (w_raw * inv_l)));
        }
        if (row < rows_valid) *reinterpret_cast<uint4*>(o + 32 * half + 8 * pc) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
  }
  if (!ok && warp == 0) {  // let copies in flight land before the shared memory is released
    for (int s = 0; s < 2; ++s)
      if (issued & (1u << s)) (void)mbar_wait(bar_stage0 + 8 * s, (st_phase >> s) & 1u);
  }
  fence_before();
  __syncthreads();
  if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tbase), "r"(512));
}

// ---------------------------------------------------------------- self-test
// One thread waits, with this kernel's bounded wait, on a barrier that nothing
// arrives at; the wait gives up after its limit and the timeout is recorded.
__global__ void selftest_wait_prefill_kernel(int32_t* dev_status) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_u32(&bar);
  asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(b));
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if (!mbar_wait(b, 0)) report_error(dev_status, KVQ_ERR_DEVICE_TIMEOUT);
}

template <int T, int BK, int BV>
cudaError_t launch_t(const PrefillArgs& a, cudaStream_t s, long long units) {
  using Geo = PfGeom<T, BK, BV>;
  auto kern = prefill_attn_kernel<T, BK, BV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<static_cast<unsigned>(units), kPfThreads, Geo::kSmem, s>>>(a);
  return cudaGetLastError();
}

template <int T>
cudaError_t launch_bits(const PrefillArgs& a, cudaStream_t s, long long units) {
  const int bk = a.cfg.bits_k, bv = a.cfg.bits_v;
  if (bk == 4 && bv == 4) return launch_t<T, 4, 4>(a, s, units);
  if (bk == 4 && bv == 2) return launch_t<T, 4, 2>(a, s, units);
  if (bk == 4 && bv == 3) return launch_t<T, 4, 3>(a, s, units);
  if (bk == 2 && bv == 4) return launch_t<T, 2, 4>(a, s, units);
  if (bk == 2 && bv == 3) return launch_t<T, 2, 3>(a, s, units);
  if (bk == 3 && bv == 4) return launch_t<T, 3, 4>(a, s, units);
  if (bk == 3 && bv == 2) return launch_t<T, 3, 2>(a, s, units);
  if (bk == 3 && bv == 3) return launch_t<T, 3, 3>(a, s, units);
  if (bk == 8 && bv == 8) return launch_t<T, 8, 8>(a, s, units);
  return launch_t<T, 2, 2>(a, s, units);
}

}  // namespace

int prefill_row_tiles(const kvq_config& cfg, int max_chunk) {
  return static_cast<int>((static_cast<long long>(max_chunk) * cfg.group_size + kRows - 1) / kRows);
}

cudaError_t launch_selftest_wait_prefill(int32_t* dev_status, cudaStream_t s) {
  selftest_wait_prefill_kernel<<<1, 1, 0, s>>>(dev_status);
  return cudaGetLastError();
}

size_t prefill_workspace_bytes(const kvq_config& cfg, int num_seqs, int max_chunk, int num_splits) {
  if (num_splits <= 1) return 0;
  const size_t units = static_cast<size_t>(num_seqs) * cfg.num_kv_heads * prefill_row_tiles(cfg, max_chunk);
  return units * num_splits * kRows * (4 + kHeadDim) * sizeof(float);
}

template <int T>
cudaError_t launch_modes(const PrefillArgs& a, cudaStream_t s, long long units) {
  if (a.num_splits <= 1) {
    PrefillArgs f = a;
    f.mode = 0;
    return launch_bits<T>(f, s, units);
  }
  PrefillArgs p = a;
  p.mode = 1;
  cudaError_t e = launch_bits<T>(p, s, units * a.num_splits);
  if (e != cudaSuccess) return e;
  p.mode = 2;
  return launch_bits<T>(p, s, units);
}

cudaError_t launch_paged_prefill(const PrefillArgs& a, cudaStream_t s) {
  const long long units = static_cast<long long>(a.num_seqs) * a.cfg.num_kv_heads * a.row_tiles;
  if (units == 0) return cudaSuccess;
  switch (a.cfg.tile_tokens) {
    case 32: return launch_modes<32>(a, s, units);
    case 64: return launch_modes<64>(a, s, units);
    default: return launch_modes<128>(a, s, units);
  }
}

}  // namespace kvq
