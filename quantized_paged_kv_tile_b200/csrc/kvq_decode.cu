// Read path: paged decode attention over the packed pages.
//
// The attention backend reads the compressed pages directly (aitrends.kr
// article 74976, "TL;DR"; glossary "attention backend").  Per (sequence,
// KV head) the g query heads are rotated once, q' = H q, and each tile t
// contributes in the rotated domain
//   score_i = s~K_i (q'' . codeK_i) + z~K_i sum_j q''_j,   q'' = q' * C~K_t
//   acc'_j += C~V_tj (sum_i p_i s~V_i codeV_ij + sum_i p_i z~V_i)
// which equals softmax(q' . K^'_i) P V^' exactly in real arithmetic.
//
// Kernels (three launches per call):
//   decode_schedule_kernel  one CTA: tiles per sequence, chunk size, the
//                           prefix of work units (sequence, KV head, chunk)
//   decode_tiles_kernel     persistent warps, one work unit at a time:
//                           per-warp double-buffered cp.async.bulk staging
//                           of whole tiles (all pages, K and V) into shared
//                           memory; scores and P.V on the legacy tensor
//                           cores (mma.sync m16n8k16, f16 -> f32) with the
//                           16 MMA rows = 8 query heads x {hi, lo} fp16
//                           halves (fp32-accurate operands at no extra MMA)
//                           and the packed codes unpacked in registers;
//                           online softmax per tile; rotated-domain partial
//   decode_merge_kernel     per (sequence, KV head): raw fp16 tail, log-sum-
//                           exp merge of the chunks, the one inverse rotation,
//                           fp16 output
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "kvq_device.cuh"

namespace kvq {

namespace {

// Partial record per (work unit, query head): m, l, two pad floats, acc[d];
// 132 floats = 528 bytes, so every record and its acc start 16-byte aligned.
constexpr int kPartFloats = 4 + kHeadDim;
constexpr int kPartAcc = 4;
constexpr int kUnitsPerSm = 32;            // work-unit budget of the automatic split
constexpr long long kWaitLimitNs = 2000000000LL;  // bounded mbarrier waits: 2 s

// ------------------------------------------------------------------ workspace
// [0]        int32 U (total work units)
// [4..]      int32 prefix[B+1]: chunks of sequences 0..b-1 (per KV head)
// then       int32 chunk[B]: tiles per chunk of each sequence
// at 256-B   float partial[U][G][4 + d]  (m, l, pad, pad, acc)
struct WsLayout {
  size_t prefix_off, chunk_off, part_off;
};
__host__ __device__ inline WsLayout ws_layout(int num_seqs) {
  WsLayout l;
  l.prefix_off = 4;
  l.chunk_off = l.prefix_off + 4 * static_cast<size_t>(num_seqs + 1);
  l.part_off = (l.chunk_off + 4 * static_cast<size_t>(num_seqs) + 255) / 256 * 256;
  return l;
}

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ long long global_ns() {
  long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
// Wait for a phase with a time bound; false on timeout.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mma16816(float d[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// Channel pair p (0..15) of lane-quad t in the K register order:
// b = 4: word p/4, nibbles (p%4, p%4+4) -> channels 32t + 8(p/4) + p%4 + {0, 4}
// b = 2: word p/8, fields (p%8, p%8+8) -> channels 32t + 16(p/8) + p%8 + {0, 8}
// b = 8: word p/2, bytes (p%2, p%2+2) -> channels 32t + 4(p/2) + p%2 + {0, 2}
template <int B>
__device__ __forceinline__ constexpr int pair_ch0(int p) {
  return B == 8 ? 4 * (p / 2) + (p % 2) : (B == 4 ? 8 * (p / 4) + (p % 4) : 16 * (p / 8) + (p % 8));
}
template <int B>
__device__ __forceinline__ constexpr int pair_gap() {
  return B == 8 ? 2 : (B == 4 ? 4 : 8);
}

// ------------------------------------------------------------------ schedule
__global__ void __launch_bounds__(1024) decode_schedule_kernel(const int32_t* seq_lens, int num_seqs, int tile_tokens,
                                                               int num_kv_heads, int num_splits, int target_units,
                                                               void* workspace) {
  __shared__ long long s_total;
  __shared__ int s_scan[1024];
  __shared__ int s_carry;
  const WsLayout wl = ws_layout(num_seqs);
  int32_t* ws_i = static_cast<int32_t*>(workspace);
  int32_t* prefix = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + wl.prefix_off);
  int32_t* chunk = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + wl.chunk_off);
  const int tid = threadIdx.x;
  if (tid == 0) {
    s_total = 0;
    s_carry = 0;
  }
  __syncthreads();
  long long part = 0;
  for (int b = tid; b < num_seqs; b += blockDim.x) part += max(seq_lens[b], 0) / tile_tokens;
  atomicAdd(reinterpret_cast<unsigned long long*>(&s_total), static_cast<unsigned long long>(part));
  __syncthreads();
  const long long total = s_total;
  long long ch_auto = 1;
  if (num_splits == 0 && total > 0)
    ch_auto = std::max(1LL, (total * num_kv_heads + target_units - 1) / target_units);
  for (int base = 0; base < num_seqs; base += blockDim.x) {
    const int b = base + tid;
    int units = 0;
    if (b < num_seqs) {
      const int f = max(seq_lens[b], 0) / tile_tokens;
      int ch;
      if (num_splits > 0) {
        const int s = min(num_splits, f);
        ch = s > 0 ? (f + s - 1) / s : 1;
      } else {
        ch = static_cast<int>(std::min<long long>(ch_auto, 1 << 30));
      }
      units = f > 0 ? (f + ch - 1) / ch : 0;
      chunk[b] = ch;
    }
    s_scan[tid] = units;
    __syncthreads();
    for (int off = 1; off < static_cast<int>(blockDim.x); off <<= 1) {  // inclusive scan
      const int v = tid >= off ? s_scan[tid - off] : 0;
      __syncthreads();
      s_scan[tid] += v;
      __syncthreads();
    }
    if (b < num_seqs) prefix[b] = s_carry + s_scan[tid] - units;
    __syncthreads();
    if (tid == blockDim.x - 1) s_carry += s_scan[tid];
    __syncthreads();
  }
  if (tid == 0) {
    prefix[num_seqs] = s_carry;
    ws_i[0] = s_carry * num_kv_heads;
  }
}

// ------------------------------------------------------------------ main decode
template <int T, int BK, int BV>
struct DecodeGeom {
  static constexpr int kPages = T / kPageTokens;
  static constexpr int kCodesK = kPageTokens * kHeadDim * BK / 8;
  static constexpr int kCodesV = kPageTokens * kHeadDim * BV / 8;
  static constexpr int kCs = kHeadDim * kPageTokens / T;        // C-slice channels per page
  static constexpr int kCsBytes = (2 * kCs + 15) / 16 * 16;
  static constexpr int kPageK = kCodesK + 64 + kCsBytes;
  static constexpr int kPageV = kCodesV + 64 + kCsBytes;
  static constexpr int kStage = kPages * (kPageK + kPageV);    // one tile, K pages then V pages
  // warps per CTA: 4, fewer when two stages per warp would not fit (8-bit codes)
  static constexpr int kWarps = 4 * (2 * kStage + 16) <= 200 * 1024 ? 4 : (2 * (2 * kStage + 16) <= 200 * 1024 ? 2 : 1);
  static constexpr int kSmem = kWarps * (2 * kStage + 16);
};

template <int T, int BK, int BV>
__global__ void __launch_bounds__(DecodeGeom<T, BK, BV>::kWarps * 32, BK == 8 ? 1 : (T == 128 ? 2 : 3))
    decode_tiles_kernel(DecodeArgs a) {
  using Geo = DecodeGeom<T, BK, BV>;
  constexpr int NP = Geo::kPages;
  constexpr int kDecWarps = Geo::kWarps;
  extern __shared__ __align__(128) unsigned char smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  unsigned char* stage_base = smem + warp * 2 * Geo::kStage;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecWarps * 2 * Geo::kStage) + 2 * warp;
  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();

  const int G = a.cfg.group_size, nh = a.cfg.num_kv_heads;
  const WsLayout wl = ws_layout(a.num_seqs);
  const int32_t* ws_i = static_cast<const int32_t*>(a.workspace);
  const int32_t* prefix = reinterpret_cast<const int32_t*>(static_cast<const char*>(a.workspace) + wl.prefix_off);
  const int32_t* chunk = reinterpret_cast<const int32_t*>(static_cast<const char*>(a.workspace) + wl.chunk_off);
  float* parts = reinterpret_cast<float*>(static_cast<char*>(a.workspace) + wl.part_off);
  const int U = ws_i[0];
  const uint8_t* kpool = static_cast<const uint8_t*>(a.k_pool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.v_pool);
  const float qscale = a.softmax_scale * kLog2e / kSqrtHeadDim;
  const bool head_live = g < G;
  uint32_t phase[2] = {0u, 0u};
  bool pending[2] = {false, false};  // copies issued into the stage and not yet waited for
  bool failed = false;

  const int total_warps = gridDim.x * kDecWarps;
  for (int u = blockIdx.x * kDecWarps + warp; u < U && !failed; u += total_warps) {
    // ---- locate the unit: sequence b (binary search), head h, chunk c
    int lo = 0, hi = a.num_seqs;  // find the largest b with nh*prefix[b] <= u
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (nh * prefix[mid] <= u) lo = mid; else hi = mid;
    }
    const int b = lo;
    const int S = prefix[b + 1] - prefix[b];
    const int r = u - nh * prefix[b];
    const int h = r / S, c = r % S;
    const int F = max(a.seq_lens[b], 0) / T;
    const int ch = chunk[b];
    const int t0 = c * ch, t1 = min(F, t0 + ch);

    // ---- rotated, scaled query: lane (g, t) holds channels 32t..32t+31 of head g
    float qs[32];
    if (head_live) {
      const __half* qp = static_cast<const __half*>(a.q) +
                         ((static_cast<size_t>(b) * nh + h) * G + g) * kHeadDim + 32 * t;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 raw = *reinterpret_cast<const uint4*>(qp + 8 * v);
        const __half2* hp = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float2 f = __half22float2(hp[k]);
          qs[8 * v + 2 * k] = f.x;
          qs[8 * v + 2 * k + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) qs[i] = 0.f;
    }
    if (a.cfg.rotation_seed != 0) {  // q' = H D_s q
#pragma unroll
      for (int i = 0; i < 32; ++i) qs[i] *= rotation_sign(a.cfg.rotation_seed, 32 * t + i);
    }
#pragma unroll
    for (int bit = 0; bit < 5; ++bit) {  // channel bits 0..4: in-register butterflies
      const int m = 1 << bit;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!(i & m)) {
          const float x = qs[i], y = qs[i | m];
          qs[i] = x + y;
          qs[i | m] = x - y;
        }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {  // channel bits 5, 6: lanes with t differing in bit k
      const int m = 1 << k;
      const bool upper = t & m;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float o = __shfl_xor_sync(kFull, qs[i], m);
        qs[i] = upper ? (o - qs[i]) : (qs[i] + o);
      }
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) qs[i] *= qscale;

    float m_run = -INFINITY, l_part = 0.f;
    float acc[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = 0.f;

    // ---- issue the first two tiles
    auto issue = [&](int tile, int st) {
      // lanes 0..NP-1 read and check the block ids of the tile's pages
      const int lb = tile * NP + lane;
      int blk = -1;
      if (lane < NP)
        blk = lb < a.max_blocks_per_seq ? a.block_tables[static_cast<size_t>(b) * a.max_blocks_per_seq + lb] : -1;
      const bool bad = lane < NP && (blk < 0 || blk >= a.num_blocks);
      if (__any_sync(kFull, bad)) {
        if (lane == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
        pending[st] = false;
        return;
      }
      if (lane == 0) mbar_arrive_expect_tx(&bars[st], NP * (Geo::kPageK + Geo::kPageV));
      __syncwarp();
      unsigned char* dst = stage_base + st * Geo::kStage;
      if (lane < NP) {
        const size_t reg = static_cast<size_t>(blk) * nh + h;
        bulk_g2s(dst + lane * Geo::kPageK, kpool + reg * Geo::kPageK, Geo::kPageK, &bars[st]);
        bulk_g2s(dst + NP * Geo::kPageK + lane * Geo::kPageV, vpool + reg * Geo::kPageV, Geo::kPageV, &bars[st]);
      }
      pending[st] = true;
    };
    if (t0 < t1) issue(t0, 0);
    if (t0 + 1 < t1) issue(t0 + 1, 1);

    for (int i = t0; i < t1; ++i) {
      const int st = (i - t0) & 1;
      if (!pending[st]) {  // tile skipped (bad block id, already reported)
        if (i + 2 < t1) issue(i + 2, st);
        continue;
      }
      if (!mbar_wait_bounded(&bars[st], phase[st])) {
        if (lane == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_TIMEOUT);
        failed = true;
        break;
      }
      phase[st] ^= 1u;
      pending[st] = false;
      const unsigned char* sK = stage_base + st * Geo::kStage;
      const unsigned char* sV = sK + NP * Geo::kPageK;

      // -- scores: D[16 rows][8 tokens] per (page, n-block); rows g / g+8 = head g hi / lo.
      // The A fragments, q'' = q' * C~K in hi/lo fp16 pairs, are built per
      // k-block from q' and the tile's C~K slice (not all held at once), and
      // sigma = sum_j q''_j is accumulated on the way.  Pages go in chunks of
      // up to 4 so that one chunk's code words and accumulators are live; the
      // chunk's scores (log2 domain, tokens 8nb + 2t, 8nb + 2t + 1 of each page)
      // are kept.
      constexpr int kPcMax = BK == 8 ? 2 : 4;
      constexpr int kPc = NP < kPcMax ? NP : kPcMax;
      float sig = 0.f;
      float sc[NP][2][2];
      float mt = -INFINITY;
      // C~K of channels 32t + c, c + 1 (c even) within the tile's page slices
      auto ck_pair = [&](int c) {
        const int ch = 32 * t + c;
        const __half2 h = *reinterpret_cast<const __half2*>(sK + (ch / Geo::kCs) * Geo::kPageK + Geo::kCodesK + 64 +
                                                            2 * (ch % Geo::kCs));
        return __half22float2(h);
      };
#pragma unroll
      for (int pc = 0; pc < NP; pc += kPc) {
        float sd[kPc][2][4];
#pragma unroll
        for (int pg = 0; pg < kPc; ++pg)
#pragma unroll
          for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int k = 0; k < 4; ++k) sd[pg][nb][k] = 0.f;
        // lane (g, t) reads its 4*BK-byte chunk (channels 32t..32t+31) of tokens g and 8+g
        uint32_t rec[kPc][2][BK];
#pragma unroll
        for (int pg = 0; pg < kPc; ++pg)
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            const unsigned char* src = sK + (pc + pg) * Geo::kPageK + (8 * nb + g) * (16 * BK) + t * (4 * BK);
            if constexpr (BK == 8) {
              const uint4 v0 = *reinterpret_cast<const uint4*>(src);
              const uint4 v1 = *reinterpret_cast<const uint4*>(src + 16);
              rec[pg][nb][0] = v0.x; rec[pg][nb][1] = v0.y; rec[pg][nb][2] = v0.z; rec[pg][nb][3] = v0.w;
              rec[pg][nb][4] = v1.x; rec[pg][nb][5] = v1.y; rec[pg][nb][6] = v1.z; rec[pg][nb][7] = v1.w;
            } else if constexpr (BK == 4) {
              const uint4 v = *reinterpret_cast<const uint4*>(src);
              rec[pg][nb][0] = v.x; rec[pg][nb][1] = v.y; rec[pg][nb][2] = v.z; rec[pg][nb][3] = v.w;
            } else {
              const uint2 v = *reinterpret_cast<const uint2*>(src);
              rec[pg][nb][0] = v.x; rec[pg][nb][1] = v.y;
            }
          }
        constexpr int kbPerWord = 8 / BK;  // k-blocks per word: 2 (b=4) or 4 (b=2)
#pragma unroll
        for (int wd = 0; wd < BK; ++wd) {
          uint32_t pr[kPc][2][16 / BK];
#pragma unroll
          for (int pg = 0; pg < kPc; ++pg)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) unpack_pairs<BK>(rec[pg][nb][wd], pr[pg][nb]);
#pragma unroll
          for (int j = 0; j < kbPerWord; ++j) {
            const int kb = wd * kbPerWord + j;
            // pairs 2kb, 2kb+1: channels (c0, c1) and (c0+1, c1+1), c0 even
            const int c0 = pair_ch0<BK>(2 * kb), c1 = c0 + pair_gap<BK>();
            const float2 ka = ck_pair(c0), kc = ck_pair(c1);
            const float x00 = qs[c0] * ka.x, x01 = qs[c0 + 1] * ka.y;
            const float x10 = qs[c1] * kc.x, x11 = qs[c1 + 1] * kc.y;
            if (pc == 0) sig += (x00 + x01) + (x10 + x11);
            const __half2 h0 = __floats2half2_rn(x00, x10), h1 = __floats2half2_rn(x01, x11);
            const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
            const uint32_t afr[4] = {h2_as_u32(h0), h2_as_u32(__floats2half2_rn(x00 - f0.x, x10 - f0.y)),
                                     h2_as_u32(h1), h2_as_u32(__floats2half2_rn(x01 - f1.x, x11 - f1.y))};
#pragma unroll
            for (int pg = 0; pg < kPc; ++pg)
#pragma unroll
              for (int nb = 0; nb < 2; ++nb) mma16816(sd[pg][nb], afr, pr[pg][nb][2 * j], pr[pg][nb][2 * j + 1]);
          }
        }
        if (pc == 0) {
          sig += __shfl_xor_sync(kFull, sig, 1);
          sig += __shfl_xor_sync(kFull, sig, 2);
        }
#pragma unroll
        for (int pg = 0; pg < kPc; ++pg) {
          const unsigned char* meta = sK + (pc + pg) * Geo::kPageK + Geo::kCodesK;
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            const uint2 mm = *reinterpret_cast<const uint2*>(meta + 4 * (8 * nb + 2 * t));
            const float2 m0 = __half22float2(u32_as_h2(mm.x)), m1 = __half22float2(u32_as_h2(mm.y));
            sc[pc + pg][nb][0] = m0.x * (sd[pg][nb][0] + sd[pg][nb][2]) + m0.y * sig;
            sc[pc + pg][nb][1] = m1.x * (sd[pg][nb][1] + sd[pg][nb][3]) + m1.y * sig;
            mt = fmaxf(mt, fmaxf(sc[pc + pg][nb][0], sc[pc + pg][nb][1]));
          }
        }
      }
      mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 2));
      const float m_new = fmaxf(m_run, mt);
      const float alpha = exp2f(m_run - m_new);
      m_run = m_new;
      l_part *= alpha;

      // -- P = p * s~V as hi/lo fp16 A fragments per page; w = sum p z~V
      uint32_t pa[NP][4];
      float wsum = 0.f;
#pragma unroll
      for (int pg = 0; pg < NP; ++pg) {
        const unsigned char* meta = sV + pg * Geo::kPageV + Geo::kCodesV;
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          const uint2 mm = *reinterpret_cast<const uint2*>(meta + 4 * (8 * nb + 2 * t));
          const float2 m0 = __half22float2(u32_as_h2(mm.x)), m1 = __half22float2(u32_as_h2(mm.y));
          const float p0 = exp2f(sc[pg][nb][0] - m_new), p1 = exp2f(sc[pg][nb][1] - m_new);
          l_part += p0 + p1;
          wsum += p0 * m0.y + p1 * m1.y;
          const float x0 = p0 * m0.x, x1 = p1 * m1.x;
          const __half2 hv = __floats2half2_rn(x0, x1);
          const float2 hf = __half22float2(hv);
          pa[pg][2 * nb] = h2_as_u32(hv);
          pa[pg][2 * nb + 1] = h2_as_u32(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
        }
      }
      wsum += __shfl_xor_sync(kFull, wsum, 1);
      wsum += __shfl_xor_sync(kFull, wsum, 2);

      // -- P V: D[16 rows][8 channels] per n-block (channels 8nv..8nv+7).  Lane
      // words 2q, 2q+1 (token pairs {2t,2t+1} and {2t+8,2t+9}) hold the n-blocks
      // kPairsV*q .. kPairsV*q + kPairsV-1; a group's accumulators are folded
      // into acc' (times C~V) as soon as all pages of the tile are in.
      constexpr int kPairsV = 16 / BV;      // n-blocks per word pair
      constexpr int kGroups = 16 / kPairsV;  // word pairs per lane (4 at b=4, 2 at b=2)
#pragma unroll
      for (int q = 0; q < kGroups; ++q) {
        float dv[kPairsV][4];
#pragma unroll
        for (int e = 0; e < kPairsV; ++e)
#pragma unroll
          for (int k = 0; k < 4; ++k) dv[e][k] = 0.f;
#pragma unroll
        for (int pg = 0; pg < NP; ++pg) {
          const uint32_t afr[4] = {pa[pg][0], pa[pg][1], pa[pg][2], pa[pg][3]};
          // words 2q and 2q+1 sit in the same 16-byte row of the lane; the whole
          // row is loaded (lanes read consecutive 16-byte rows: no bank conflict)
          const uint4 row = *reinterpret_cast<const uint4*>(sV + pg * Geo::kPageV + (((2 * q) >> 2) * 32 + lane) * 16);
          const uint32_t w0 = (q & 1) ? row.z : row.x, w1 = (q & 1) ? row.w : row.y;
          uint32_t p0[kPairsV], p1[kPairsV];
          unpack_pairs<BV>(w0, p0);
          unpack_pairs<BV>(w1, p1);
#pragma unroll
          for (int e = 0; e < kPairsV; ++e) mma16816(dv[e], afr, p0[e], p1[e]);
        }
#pragma unroll
        for (int e = 0; e < kPairsV; ++e) {
          const int nv = kPairsV * q + e;
          const int c0 = 8 * nv + 2 * t;
          const __half2 cvh = *reinterpret_cast<const __half2*>(sV + (c0 / Geo::kCs) * Geo::kPageV + Geo::kCodesV +
                                                                64 + 2 * (c0 % Geo::kCs));
          const float2 cv = __half22float2(cvh);
          acc[2 * nv] = alpha * acc[2 * nv] + cv.x * (dv[e][0] + dv[e][2] + wsum);
          acc[2 * nv + 1] = alpha * acc[2 * nv + 1] + cv.y * (dv[e][1] + dv[e][3] + wsum);
        }
      }
      __syncwarp();
      if (i + 2 < t1) issue(i + 2, st);
    }
    if (failed) break;

    // ---- partial of this unit
    float l_tot = l_part + __shfl_xor_sync(kFull, l_part, 1);
    l_tot += __shfl_xor_sync(kFull, l_tot, 2);
    if (head_live) {
      float* part = parts + (static_cast<size_t>(u) * G + g) * kPartFloats;
      if (t == 0) {
        part[0] = m_run;
        part[1] = l_tot;
      }
#pragma unroll
      for (int nv = 0; nv < 16; ++nv) {
        const int c0 = 8 * nv + 2 * t;
        *reinterpret_cast<float2*>(part + kPartAcc + c0) = make_float2(acc[2 * nv], acc[2 * nv + 1]);
      }
    }
  }
  if (failed) {  // let copies already in flight land before the CTA's shared memory is released
    for (int st = 0; st < 2; ++st)
      if (pending[st]) (void)mbar_wait_bounded(&bars[st], phase[st]);
  }
}

// ------------------------------------------------------------------ self-test
// The decode kernel's bounded wait on a barrier that nothing arrives at.
__global__ void selftest_wait_decode_kernel(int32_t* dev_status) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if (!mbar_wait_bounded(&bar, 0)) report_error(dev_status, KVQ_ERR_DEVICE_TIMEOUT);
}

// ------------------------------------------------------------------ merge
constexpr int kMergeThreads = 256;

template <int T>
struct __align__(16) MergeSmem {
  float qraw[kMaxGroup][kHeadDim];
  float sc[kMaxGroup][T];
  float tl[kMaxGroup][kHeadDim];                 // raw-domain tail accumulator
  float red[kMergeThreads / 32][kHeadDim];       // per-warp partial sums of one head
  float big_m[kMaxGroup], inv_l[kMaxGroup], et[kMaxGroup], mt[kMaxGroup], lt[kMaxGroup];
};

// One CTA of 256 threads per (sequence, KV head): raw fp16 tail, log-sum-
// exp merge of the chunk partials (warps split the chunks, lanes own four
// channels), the inverse rotation of the merged accumulator, fp16 output.
template <int T>
__global__ void __launch_bounds__(kMergeThreads) decode_merge_kernel(DecodeArgs a) {
  __shared__ MergeSmem<T> sm;
  constexpr int kWarps = kMergeThreads / 32;
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.cfg.group_size, nh = a.cfg.num_kv_heads;
  const int L = max(a.seq_lens[b], 0);
  const int F = L / T, tau = L - F * T;
  const WsLayout wl = ws_layout(a.num_seqs);
  const int32_t* prefix = reinterpret_cast<const int32_t*>(static_cast<const char*>(a.workspace) + wl.prefix_off);
  const float* parts = reinterpret_cast<const float*>(static_cast<const char*>(a.workspace) + wl.part_off);
  const int S = prefix[b + 1] - prefix[b];
  const size_t ubase = static_cast<size_t>(nh) * prefix[b] + static_cast<size_t>(h) * S;
  const float qscale = a.softmax_scale * kLog2e;
  const __half* q = static_cast<const __half*>(a.q) + (static_cast<size_t>(b) * nh + h) * G * kHeadDim;
  const __half* kt = static_cast<const __half*>(a.k_tail) + (static_cast<size_t>(b) * nh + h) * T * kHeadDim;
  const __half* vt = static_cast<const __half*>(a.v_tail) + (static_cast<size_t>(b) * nh + h) * T * kHeadDim;

  // 1. raw tail: scores (thread = token), softmax (warp = head), P V (thread = channel)
  for (int idx = tid; idx < G * kHeadDim; idx += kMergeThreads)
    sm.qraw[idx / kHeadDim][idx % kHeadDim] = __half2float(q[idx]) * qscale;
  __syncthreads();
  for (int i = tid; i < tau; i += kMergeThreads) {
    float dot[kMaxGroup];
#pragma unroll
    for (int hh = 0; hh < kMaxGroup; ++hh) dot[hh] = 0.f;
    for (int c = 0; c < kHeadDim; ++c) {
      const float kv = __half2float(kt[i * kHeadDim + c]);
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh)
        if (hh < G) dot[hh] += sm.qraw[hh][c] * kv;
    }
    for (int hh = 0; hh < G; ++hh) sm.sc[hh][i] = dot[hh];
  }
  __syncthreads();
  for (int hh = warp; hh < G; hh += kWarps) {
    float m = -INFINITY;
    for (int i = lane; i < tau; i += 32) m = fmaxf(m, sm.sc[hh][i]);
    m = warp_max(m);
    float ps = 0.f;
    for (int i = lane; i < tau; i += 32) {
      const float p = exp2f(sm.sc[hh][i] - m);
      sm.sc[hh][i] = p;
      ps += p;
    }
    ps = warp_sum(ps);
    // merge statistics over the chunks: the warp's lanes stride over them
    float mm = m;
    for (int s = lane; s < S; s += 32) {
      const float* pp = parts + ((ubase + s) * G + hh) * kPartFloats;
      if (pp[1] > 0.f) mm = fmaxf(mm, pp[0]);
    }
    mm = warp_max(mm);
    float ll = 0.f;
    for (int s = lane; s < S; s += 32) {
      const float* pp = parts + ((ubase + s) * G + hh) * kPartFloats;
      if (pp[1] > 0.f) ll += pp[1] * exp2f(pp[0] - mm);
    }
    ll = warp_sum(ll);
    if (lane == 0) {
      const float et = ps > 0.f ? exp2f(m - mm) : 0.f;
      const float l = ll + ps * et;
      sm.big_m[hh] = mm;
      sm.et[hh] = et;
      sm.inv_l[hh] = l > 0.f ? 1.f / l : 0.f;
    }
  }
  __syncthreads();  // tail weights in sm.sc are read by every thread below
  for (int idx = tid; idx < G * kHeadDim; idx += kMergeThreads) {
    const int hh = idx / kHeadDim, c = idx % kHeadDim;
    float at = 0.f;
    for (int i = 0; i < tau; ++i) at += sm.sc[hh][i] * __half2float(vt[i * kHeadDim + c]);
    sm.tl[hh][c] = at;
  }
  __syncthreads();

  // 2. per head: warps split the chunks, lane owns channels 4*lane .. 4*lane+3
  __half* out = static_cast<__half*>(a.out) + (static_cast<size_t>(b) * nh + h) * G * kHeadDim;
  for (int hh = 0; hh < G; ++hh) {
    const float mm = sm.big_m[hh];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int s = warp; s < S; s += kWarps) {
      const float* pp = parts + ((ubase + s) * G + hh) * kPartFloats;
      const float2 ml = *reinterpret_cast<const float2*>(pp);
      const float4 v = *reinterpret_cast<const float4*>(pp + kPartAcc + 4 * lane);
      if (ml.y > 0.f) {
        const float wgt = exp2f(ml.x - mm);
        acc.x += wgt * v.x;
        acc.y += wgt * v.y;
        acc.z += wgt * v.z;
        acc.w += wgt * v.w;
      }
    }
    *reinterpret_cast<float4*>(&sm.red[warp][4 * lane]) = acc;
    __syncthreads();
    if (warp == 0) {
      float v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float x = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) x += sm.red[w][4 * lane + k];
        v[k] = x;
      }
      fwht128_warp(v, lane);  // the one inverse rotation (H = H^T = H^-1)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int c = 4 * lane + k;
        out[hh * kHeadDim + c] = __float2half_rn(
            (v[k] / kSqrtHeadDim * rotation_sign(a.cfg.rotation_seed, c) + sm.et[hh] * sm.tl[hh][c]) * sm.inv_l[hh]);
      }
    }
    __syncthreads();
  }
}

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int T, int BK, int BV>
cudaError_t launch_tiles_t(const DecodeArgs& a, cudaStream_t s, int grid) {
  using Geo = DecodeGeom<T, BK, BV>;
  auto kern = decode_tiles_kernel<T, BK, BV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::kSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Geo::kWarps * 32, Geo::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<grid * std::max(per_sm, 1), Geo::kWarps * 32, Geo::kSmem, s>>>(a);
  return cudaGetLastError();
}

template <int T>
cudaError_t launch_tiles_bits(const DecodeArgs& a, cudaStream_t s, int grid) {
  if (a.cfg.bits_k == 4 && a.cfg.bits_v == 4) return launch_tiles_t<T, 4, 4>(a, s, grid);
  if (a.cfg.bits_k == 4 && a.cfg.bits_v == 2) return launch_tiles_t<T, 4, 2>(a, s, grid);
  if (a.cfg.bits_k == 2 && a.cfg.bits_v == 4) return launch_tiles_t<T, 2, 4>(a, s, grid);
  if (a.cfg.bits_k == 8 && a.cfg.bits_v == 8) return launch_tiles_t<T, 8, 8>(a, s, grid);
  return launch_tiles_t<T, 2, 2>(a, s, grid);
}

template <int T>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t s) {
  const int sms = device_sms();
  decode_schedule_kernel<<<1, 1024, 0, s>>>(a.seq_lens, a.num_seqs, T, a.cfg.num_kv_heads, a.num_splits_fixed,
                                            kUnitsPerSm * sms, a.workspace);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = launch_tiles_bits<T>(a, s, sms);
  if (e != cudaSuccess) return e;
  dim3 g2(a.cfg.num_kv_heads, a.num_seqs);
  decode_merge_kernel<T><<<g2, kMergeThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t decode_workspace_bytes(const kvq_config& cfg, int num_seqs, int num_splits, int num_sms) {
  const WsLayout wl = ws_layout(num_seqs);
  const size_t units = num_splits > 0
                           ? static_cast<size_t>(num_seqs) * cfg.num_kv_heads * num_splits
                           : static_cast<size_t>(kUnitsPerSm) * num_sms + static_cast<size_t>(num_seqs) * cfg.num_kv_heads;
  return wl.part_off + units * cfg.group_size * kPartFloats * sizeof(float);
}

cudaError_t launch_selftest_wait_decode(int32_t* dev_status, cudaStream_t s) {
  selftest_wait_decode_kernel<<<1, 1, 0, s>>>(dev_status);
  return cudaGetLastError();
}

cudaError_t launch_paged_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.num_seqs == 0) return cudaSuccess;
  switch (a.cfg.tile_tokens) {
    case 32: return launch_decode_t<32>(a, s);
    case 64: return launch_decode_t<64>(a, s);
    default: return launch_decode_t<128>(a, s);
  }
}

}  // namespace kvq
