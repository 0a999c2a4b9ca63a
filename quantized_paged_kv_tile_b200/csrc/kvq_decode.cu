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
// Kernels (two launches per call):
//   decode_schedule_kernel  one CTA: tiles per sequence, chunk size, the
//                           prefix of work units (sequence, KV head, chunk);
//                           resets the unit queue and the arrival counters
//   decode_tiles_kernel     persistent warps taking work units from a queue:
//                           per-warp double-buffered cp.async.bulk staging
//                           of whole tiles (all pages, K and V) into shared
//                           memory; scores and P.V on the legacy tensor
//                           cores (mma.sync m16n8k16, f16 -> f32) with the
//                           16 MMA rows = 8 query heads x {hi, lo} fp16
//                           halves (fp32-accurate operands at no extra MMA)
//                           and the packed codes unpacked in registers;
//                           online softmax per tile; rotated-domain partial.
//                           The unit with chunk 0 of a (sequence, KV head)
//                           also runs the raw fp16 tail; the last of its
//                           units to finish merges the partials by
//                           log-sum-exp, applies the one inverse rotation and
//                           writes the fp16 output.
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
constexpr int kTailScratch = 13 * 1024;  // warp scratch: the tail's staged V rows; the merge's weights and staging
// work-unit budget of the automatic split, per SM: about two units per
// resident warp at T <= 64 (12 warps per SM), four at T = 128 (8 warps)
__host__ __device__ constexpr int units_per_sm(int T) { return T == 128 ? 32 : 24; }
constexpr long long kWaitLimitNs = 2000000000LL;  // bounded mbarrier waits: 2 s

// ------------------------------------------------------------------ workspace
// [0]        int32 U (total work units)
// [4]        int32 next unit to hand out (dynamic schedule)
// [8]        int32 CTAs finished (fused serving step)
// [16..]     int32 prefix[B+1]: chunks of the sequences before position i of
//            the dispatch order (per KV head)
// then       int32 chunk[B]: tiles per chunk of each sequence
// then       int32 order[B]: the sequence at position i of the dispatch order
// then       int32 rank[B]: the position of sequence b in it
// then       int32 arrivals[B][H]: finished units of each (sequence, KV head)
// at 256-B   float tails[B][H][G][4 + d]  (m, l, pad, pad, acc) of the raw tail
// then       float partial[U][G][4 + d]  (m, l, pad, pad, acc) of the units
// then       int32 group[U]: finished chunks of each merge group, at the
//            slot of the group's first unit
struct WsLayout {
  size_t prefix_off, chunk_off, order_off, rank_off, arrive_off, tail_off, part_off;
};
__host__ __device__ inline WsLayout ws_layout(int num_seqs, int num_heads, int group) {
  WsLayout l;
  l.prefix_off = 16;
  l.chunk_off = l.prefix_off + 4 * static_cast<size_t>(num_seqs + 1);
  l.order_off = l.chunk_off + 4 * static_cast<size_t>(num_seqs);
  l.rank_off = l.order_off + 4 * static_cast<size_t>(num_seqs);
  l.arrive_off = l.rank_off + 4 * static_cast<size_t>(num_seqs);
  l.tail_off = (l.arrive_off + 4 * static_cast<size_t>(num_seqs) * num_heads + 255) / 256 * 256;
  l.part_off = l.tail_off + static_cast<size_t>(num_seqs) * num_heads * group * kPartFloats * sizeof(float);
  return l;
}

__host__ __device__ inline int32_t* group_counters(float* parts, size_t units, int group) {
  return reinterpret_cast<int32_t*>(parts + units * group * kPartFloats);
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
// b = 3: pair p = channels 32t + p + {0, 16} (codes at bits 3p and 3p + 48 of the lane's 96)
template <int B>
__device__ __forceinline__ constexpr int pair_ch0(int p) {
  return B == 3 ? p : (B == 8 ? 4 * (p / 2) + (p % 2) : (B == 4 ? 8 * (p / 4) + (p % 4) : 16 * (p / 8) + (p % 8)));
}
template <int B>
__device__ __forceinline__ constexpr int pair_gap() {
  return B == 3 ? 16 : (B == 8 ? 2 : (B == 4 ? 4 : 8));
}

// 3-bit field k (compile-time after unrolling) of a little-endian run of
// 32-bit words: bits 3k .. 3k + 2, possibly straddling two words
template <int N>
__device__ __forceinline__ uint32_t field3(const uint32_t (&w)[N], int k) {
  const int o = 3 * k, i = o >> 5, sh = o & 31;
  if (sh <= 29) return (w[i] >> sh) & 7u;
  return __funnelshift_r(w[i], w[i + 1], sh) & 7u;
}
__device__ __forceinline__ float max3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// two codes as an fp16 pair of exact small integers (low half `lo`)
__device__ __forceinline__ uint32_t code_pair_f16(uint32_t lo, uint32_t hi) {
  return h2_as_u32(__hsub2(u32_as_h2(lo | (hi << 16) | 0x64006400u), __float2half2_rn(1024.f)));
}

// ------------------------------------------------------------------ schedule
// Work units of the automatic (or fixed) split: chunk sizes, the dispatch
// order and its unit prefix, and the counters reset.  With up to 1024
// sequences they are dispatched longest first (a bitonic sort of the tile
// counts, ties by index), so the queue ends on short units and the warps
// finish together; the order does not change any result (each pair's records
// are merged in chunk order).
__global__ void __launch_bounds__(1024) decode_schedule_kernel(const int32_t* seq_lens, int num_seqs, int tile_tokens,
                                                               int num_kv_heads, int group, int num_splits,
                                                               int target_units, void* workspace) {
  __shared__ long long s_total;
  __shared__ int s_warp[32];
  __shared__ int s_key[1024];
  __shared__ int s_idx[1024];
  __shared__ int s_carry;
  const WsLayout wl = ws_layout(num_seqs, num_kv_heads, group);
  int32_t* ws_i = static_cast<int32_t*>(workspace);
  int32_t* prefix = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + wl.prefix_off);
  int32_t* chunk = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + wl.chunk_off);
  int32_t* order = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + wl.order_off);
  int32_t* rank = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + wl.rank_off);
  int32_t* arrivals = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + wl.arrive_off);
  const int tid = threadIdx.x;
  // the arrival counters and the unit queue start at zero on every call
  for (int i = tid; i < num_seqs * num_kv_heads; i += blockDim.x) arrivals[i] = 0;
  if (tid == 0) ws_i[1] = 0;
  if (tid == 0) {
    s_total = 0;
    s_carry = 0;
  }
  __syncthreads();
  // full tiles per sequence, read once (sequences past the block size are
  // read again below, in the order given)
  const bool sorted = num_seqs <= static_cast<int>(blockDim.x);
  const int f_own = tid < num_seqs ? max(seq_lens[tid], 0) / tile_tokens : -1;
  long long part = f_own > 0 ? f_own : 0;
  for (int b = tid + blockDim.x; b < num_seqs; b += blockDim.x) part += max(seq_lens[b], 0) / tile_tokens;
  atomicAdd(reinterpret_cast<unsigned long long*>(&s_total), static_cast<unsigned long long>(part));
  // dispatch order: longest first when the sequences fit one sort, else as given
  if (sorted) {
    s_key[tid] = f_own;
    s_idx[tid] = tid;
    int n = 1;  // the sort spans the next power of two of the sequence count
    while (n < num_seqs) n <<= 1;
    __syncthreads();
    for (int k = 2; k <= n; k <<= 1) {
      for (int jj = k >> 1; jj > 0; jj >>= 1) {
        const int p = tid ^ jj;
        if (p > tid) {
          // descending by key, ascending by index on ties, in the (tid & k) == 0 halves
          const bool first_wins = s_key[tid] > s_key[p] || (s_key[tid] == s_key[p] && s_idx[tid] < s_idx[p]);
          if (((tid & k) == 0) != first_wins) {
            const int tk = s_key[tid], ti = s_idx[tid];
            s_key[tid] = s_key[p];
            s_idx[tid] = s_idx[p];
            s_key[p] = tk;
            s_idx[p] = ti;
          }
        }
        __syncthreads();
      }
    }
    if (tid < num_seqs) {
      order[tid] = s_idx[tid];
      rank[s_idx[tid]] = tid;
    }
  } else {
    for (int b = tid; b < num_seqs; b += blockDim.x) {
      order[b] = b;
      rank[b] = b;
    }
  }
  __syncthreads();
  const long long total = s_total;
  long long ch_auto = 1;
  if (num_splits == 0 && total > 0)
    ch_auto = std::max(1LL, (total * num_kv_heads + target_units - 1) / target_units);
  for (int base = 0; base < num_seqs; base += blockDim.x) {
    const int i = base + tid;  // position in the dispatch order
    int units = 0;
    if (i < num_seqs) {
      const int b = sorted ? s_idx[i] : i;
      const int f = sorted ? s_key[i] : max(seq_lens[b], 0) / tile_tokens;
      int ch;
      if (num_splits > 0) {
        const int sp = min(num_splits, f);
        ch = sp > 0 ? (f + sp - 1) / sp : 1;
      } else {
        ch = static_cast<int>(std::min<long long>(ch_auto, 1 << 30));
      }
      // every (sequence, KV head) gets a unit, even with no full tile (its
      // records say so; the raw tail and the merge are separate units)
      units = f > 0 ? (f + ch - 1) / ch : 1;
      chunk[b] = ch;
    }
    // inclusive scan of units over the block: within warps by shuffles, then
    // over the warp totals
    const int lane = tid & 31, wid = tid >> 5, nw = blockDim.x >> 5;
    int incl = units;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) s_warp[wid] = incl;
    __syncthreads();
    if (wid == 0) {
      int w = lane < nw ? s_warp[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int v = __shfl_up_sync(kFull, w, off);
        if (lane >= off) w += v;
      }
      if (lane < nw) s_warp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    incl += (wid > 0 ? s_warp[wid - 1] : 0);
    if (i < num_seqs) prefix[i] = s_carry + incl - units;
    __syncthreads();
    if (tid == blockDim.x - 1) s_carry += incl;
    __syncthreads();
  }
  if (tid == 0) {
    prefix[num_seqs] = s_carry;
    ws_i[0] = s_carry * num_kv_heads;
  }
  // the merge-group counters after this call's partial records start at zero
  const size_t units = static_cast<size_t>(s_carry) * num_kv_heads;
  int32_t* gcount = group_counters(reinterpret_cast<float*>(static_cast<char*>(workspace) + wl.part_off), units, group);
  for (size_t i = tid; i < units; i += blockDim.x) gcount[i] = 0;
}

// ------------------------------------------------------------------ raw tail and merge
__device__ __forceinline__ float ld_cg(const float* p) { return __ldcg(p); }
__device__ __forceinline__ float4 ld_cg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }

// One warp, serving step: the step's K and V rows of (sequence b, KV head h)
// into tail row (L - 1) mod T, L the length after the step.  A token that
// completes a tile (L mod T == 0) would have to be quantized into pages, which
// this launch does not do: it is reported and not written.
template <int T>
__device__ void step_append_warp(const DecodeArgs& a, int b, int h, int L, int lane) {
  if (L % T == 0) {
    if (lane == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
    return;
  }
  const size_t bh = static_cast<size_t>(b) * a.cfg.num_kv_heads + h;
  const size_t row = (bh * T + (L - 1) % T) * kHeadDim;
  const uint2* nk = reinterpret_cast<const uint2*>(static_cast<const __half*>(a.new_k) + bh * kHeadDim);
  const uint2* nv = reinterpret_cast<const uint2*>(static_cast<const __half*>(a.new_v) + bh * kHeadDim);
  uint2* tk = reinterpret_cast<uint2*>(const_cast<__half*>(static_cast<const __half*>(a.k_tail)) + row);
  uint2* tv = reinterpret_cast<uint2*>(const_cast<__half*>(static_cast<const __half*>(a.v_tail)) + row);
  tk[lane] = nk[lane];
  tv[lane] = nv[lane];
  __syncwarp();
}

// Four 8x8 fp16 matrices from shared memory, transposed: lanes 8i..8i+7 give
// the row addresses of matrix i; register i of lane (g, t) receives elements
// (2t, g) and (2t + 1, g) of matrix i (the m16n8k16 B-fragment order).
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
constexpr int kTailRowBytes = 2 * kHeadDim + 16;  // staged V row, padded: 8 rows hit 8 distinct bank groups
static_assert(16 * kTailRowBytes <= kTailScratch, "16 staged tail rows fit the warp scratch");

// One warp: the raw fp16 tail (tau < T tokens) of (sequence b, KV head h)
// for its g query heads, in the original domain, on the tensor cores
// (mma.sync m16n8k16, rows = query heads), 16 tokens at a time with a running
// (online) softmax per head.  Scores: q and the raw K rows are fp16, so the
// products are exact and sum in fp32; lane (g, t) loads 16-byte runs of q and
// K, and k-block 2j + u takes channels 32j + 8t + 4u + {0, 1} (fragment
// columns 2t, 2t + 1) and 32j + 8t + 4u + {2, 3} (columns 2t + 8, 2t + 9) on
// both sides.  P V: the score fragments are the A fragments of P (rows g /
// g + 8 = hi / lo fp16 halves of p), V comes through shared memory as
// transposed 8x8 fp16 tiles.  The loop body is emitted once, so the code stays
// small next to the tile loop.  Writes the tail record (m, l, acc) of every
// query head; scratch: 16 padded V rows (4352 bytes) of the warp's shared
// memory, whose copies must all have landed.
template <int T>
__device__ __forceinline__ void decode_tail_warp(const DecodeArgs& a, int b, int h, int tau, float* tails, float* scratch, int lane) {
  const int G = a.cfg.group_size, nh = a.cfg.num_kv_heads;
  const int g = lane >> 2, t = lane & 3;
  const float qscale = a.softmax_scale * kLog2e;
  const size_t bh = static_cast<size_t>(b) * nh + h;
  float* rec = tails + bh * G * kPartFloats;
  if (tau <= 0) {
    for (int hh = 0; hh < G; ++hh) {
      if (lane == 0) {
        rec[hh * kPartFloats] = -INFINITY;
        rec[hh * kPartFloats + 1] = 0.f;
      }
      *reinterpret_cast<float4*>(rec + hh * kPartFloats + kPartAcc + 4 * lane) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  const bool live = g < G;
  uint4 qa[4];
  {
    const __half* qrow = static_cast<const __half*>(a.q) + (bh * G + (live ? g : 0)) * kHeadDim + 8 * t;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      qa[j] = live ? *reinterpret_cast<const uint4*>(qrow + 32 * j) : make_uint4(0u, 0u, 0u, 0u);
  }
  const __half* kt = static_cast<const __half*>(a.k_tail) + bh * T * kHeadDim;
  const __half* vt = static_cast<const __half*>(a.v_tail) + bh * T * kHeadDim;
  unsigned char* vs = reinterpret_cast<unsigned char*>(scratch);
  // ldmatrix lane 8i + r: row r of matrix i = token r + 8 (i & 1), channels 8 (nv + (i >> 1)) ..
  const uint32_t lane_addr = smem_u32(vs) + ((lane & 7) + 8 * ((lane >> 3) & 1)) * kTailRowBytes + 16 * (lane >> 4);

  float m = -INFINITY, l = 0.f;  // running max and this lane's share of the sum, head g
  float acc[16][4];
#pragma unroll
  for (int nv = 0; nv < 16; ++nv)
#pragma unroll
    for (int k = 0; k < 4; ++k) acc[nv][k] = 0.f;
#pragma unroll 1
  for (int t0 = 0; t0 < tau; t0 += 16) {
    // stage V rows t0 .. t0 + 15 (zeros past the tail: p is 0 there, and
    // 0 times a stale non-finite value would not be); the loads are in
    // flight while the scores are computed
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int idx = lane + 32 * k, row = idx >> 4, c16 = idx & 15;
      const int tk = t0 + row;
      const uint4 v = tk < tau ? *reinterpret_cast<const uint4*>(vt + static_cast<size_t>(tk) * kHeadDim + 8 * c16)
                               : make_uint4(0u, 0u, 0u, 0u);
      *reinterpret_cast<uint4*>(vs + row * kTailRowBytes + 16 * c16) = v;
    }
    // scores of tokens t0 + 8e + 2t, t0 + 8e + 2t + 1 (e = 0, 1) for head g
    float sc[2][2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int tk = t0 + 8 * e + g;
      uint4 kr[4];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        kr[j] = tk < tau ? *reinterpret_cast<const uint4*>(kt + static_cast<size_t>(tk) * kHeadDim + 32 * j + 8 * t)
                         : make_uint4(0u, 0u, 0u, 0u);
      float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t a0[4] = {qa[j].x, 0u, qa[j].y, 0u};
        const uint32_t a1[4] = {qa[j].z, 0u, qa[j].w, 0u};
        mma16816(d, a0, kr[j].x, kr[j].y);
        mma16816(d, a1, kr[j].z, kr[j].w);
      }
      const int i0 = t0 + 8 * e + 2 * t;
      sc[e][0] = i0 < tau ? d[0] * qscale : -INFINITY;
      sc[e][1] = i0 + 1 < tau ? d[1] * qscale : -INFINITY;
    }
    float cm = fmaxf(fmaxf(sc[0][0], sc[0][1]), fmaxf(sc[1][0], sc[1][1]));
    cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 1));
    cm = fmaxf(cm, __shfl_xor_sync(kFull, cm, 2));
    const float m_new = fmaxf(m, cm);  // finite: token t0 is in the tail
    const float alpha = exp2f(m - m_new);
    m = m_new;
    l *= alpha;
#pragma unroll
    for (int nv = 0; nv < 16; ++nv)
#pragma unroll
      for (int k = 0; k < 4; ++k) acc[nv][k] *= alpha;
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const float p = sc[e][k] == -INFINITY ? 0.f : exp2f(sc[e][k] - m_new);
        sc[e][k] = p;
        l += p;
      }
    uint32_t pa[4];
    {
      const __half2 hx = __floats2half2_rn(sc[0][0], sc[0][1]), hy = __floats2half2_rn(sc[1][0], sc[1][1]);
      const float2 fx = __half22float2(hx), fy = __half22float2(hy);
      pa[0] = h2_as_u32(hx);
      pa[1] = h2_as_u32(__floats2half2_rn(sc[0][0] - fx.x, sc[0][1] - fx.y));
      pa[2] = h2_as_u32(hy);
      pa[3] = h2_as_u32(__floats2half2_rn(sc[1][0] - fy.x, sc[1][1] - fy.y));
    }
    __syncwarp();
#pragma unroll
    for (int nv = 0; nv < 16; nv += 2) {
      uint32_t bf[4];
      ldsm_x4_trans(lane_addr + 16 * nv, bf);
      mma16816(acc[nv], pa, bf[0], bf[1]);
      mma16816(acc[nv + 1], pa, bf[2], bf[3]);
    }
  }
  l += __shfl_xor_sync(kFull, l, 1);
  l += __shfl_xor_sync(kFull, l, 2);
  if (live) {
    float* r = rec + g * kPartFloats;
    if (t == 0) {
      r[0] = m;
      r[1] = l;
    }
#pragma unroll
    for (int nv = 0; nv < 16; ++nv)
      *reinterpret_cast<float2*>(r + kPartAcc + 8 * nv + 2 * t) =
          make_float2(acc[nv][0] + acc[nv][2], acc[nv][1] + acc[nv][3]);
  }
  __syncwarp();
}

// Log-sum-exp merge of n partial records of (sequence b, KV head h) by one
// warp: the records at unit slots first + s * stride (s < n), written by
// other warps and read through L2.  Two levels keep every merge short: the
// chunks of a (sequence, KV head) form groups of kMergeGroup consecutive
// chunks; the last chunk of a group to finish merges the group into a record
// at the group's first slot (final = false), and the last group to finish
// merges those records with the raw tail record, applies the one inverse
// rotation of the rotated-domain accumulator and writes the fp16 output
// (final = true; a single group goes straight to this step).  The G query
// heads go together while records are read: the maxima (lanes stride over
// the records), each record's weight into the scratch, then the weighted sums
// with R records x G heads (about 16) loads in flight per lane (lane L owns
// channels 4L .. 4L+3 of every head).  The output (inverse rotation, tail,
// 1/l) then runs as one loop over the heads from the scratch, which keeps the
// code small: the tile loop of the warps that share the SM stays in the
// instruction cache.
// Scratch layout (bytes): [0, 4096) weights of kBlock records, then the
// sums [G][32 lanes] float4, the tail accumulators [G][32] float4, and
// (et, 1/l) per head.
constexpr int kMergeGroup = 16;
constexpr int kMergeWBytes = 4096;
template <int G>
__device__ __forceinline__ void decode_merge_warp_g(const DecodeArgs& a, int b, int h, int n_rec, size_t first,
                                                 int stride, bool final, float* parts, const float* tails,
                                                 float* scratch, int lane) {
  constexpr int R = 16 / G > 1 ? 16 / G : 1;     // records per round
  constexpr int kBlock = kMergeWBytes / 4 / G;   // records whose weights fit the scratch
  static_assert(kMergeWBytes + 2 * G * 512 + 8 * G <= kTailScratch, "merge scratch");
  float* wsc = scratch;
  float4* acc_s = reinterpret_cast<float4*>(reinterpret_cast<unsigned char*>(scratch) + kMergeWBytes);
  float4* tail_s = acc_s + G * 32;
  float* scal = reinterpret_cast<float*>(tail_s + G * 32);
  const int nh = a.cfg.num_kv_heads;
  const size_t bh = static_cast<size_t>(b) * nh + h;
  const float* trec = tails + bh * G * kPartFloats;
  auto rec = [&](int s, int hh) { return parts + ((first + static_cast<size_t>(s) * stride) * G + hh) * kPartFloats; };
  float mm[G], ll[G], mt[G], lt[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    mt[hh] = -INFINITY;
    lt[hh] = 0.f;
    if (final) {
      mt[hh] = ld_cg(trec + hh * kPartFloats);
      lt[hh] = ld_cg(trec + hh * kPartFloats + 1);
      tail_s[hh * 32 + lane] = ld_cg4(trec + hh * kPartFloats + kPartAcc + 4 * lane);
    }
    mm[hh] = lt[hh] > 0.f ? mt[hh] : -INFINITY;
    ll[hh] = 0.f;
  }
  for (int s = lane; s < n_rec; s += 32) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      const float2 ml = __ldcg(reinterpret_cast<const float2*>(rec(s, hh)));
      if (ml.y > 0.f) mm[hh] = fmaxf(mm[hh], ml.x);
    }
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh) mm[hh] = warp_max(mm[hh]);
  float4 acc[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) acc[hh] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < n_rec; s0 += kBlock) {
    const int n = min(kBlock, n_rec - s0);
    __syncwarp();
    for (int s = lane; s < n; s += 32) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float2 ml = __ldcg(reinterpret_cast<const float2*>(rec(s0 + s, hh)));
        const float w = ml.y > 0.f ? exp2f(ml.x - mm[hh]) : 0.f;
        ll[hh] += w * ml.y;
        wsc[s * G + hh] = w;
      }
    }
    __syncwarp();
    for (int s = 0; s < n; s += R) {
      float4 v[R][G];
#pragma unroll
      for (int k = 0; k < R; ++k)
#pragma unroll
        for (int hh = 0; hh < G; ++hh)
          v[k][hh] = s + k < n ? ld_cg4(rec(s0 + s + k, hh) + kPartAcc + 4 * lane) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < R; ++k)
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
          const float w = s + k < n ? wsc[(s + k) * G + hh] : 0.f;
          acc[hh].x += w * v[k][hh].x;
          acc[hh].y += w * v[k][hh].y;
          acc[hh].z += w * v[k][hh].z;
          acc[hh].w += w * v[k][hh].w;
        }
    }
  }
  if (!final) {  // the group's record (m, l, acc), at its first slot, whose reads are all done
    __syncwarp();
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float* r = rec(0, hh);
      const float l = warp_sum(ll[hh]);
      if (lane == 0) {
        r[0] = mm[hh];
        r[1] = l;
      }
      *reinterpret_cast<float4*>(r + kPartAcc + 4 * lane) = acc[hh];
    }
    __syncwarp();
    return;
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    acc_s[hh * 32 + lane] = acc[hh];
    const float l = warp_sum(ll[hh]);
    const float et = lt[hh] > 0.f ? exp2f(mt[hh] - mm[hh]) : 0.f;
    const float ltot = l + lt[hh] * et;
    if (lane == 0) {
      scal[2 * hh] = et;
      scal[2 * hh + 1] = ltot > 0.f ? 1.f / ltot : 0.f;
    }
  }
  __syncwarp();
  __half* out = static_cast<__half*>(a.out) + bh * G * kHeadDim;
  const uint32_t seed = a.cfg.rotation_seed;
  float sg[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) sg[k] = rotation_sign(seed, 4 * lane + k) / kSqrtHeadDim;
#pragma unroll 1
  for (int hh = 0; hh < G; ++hh) {
    const float4 va = acc_s[hh * 32 + lane], tl = tail_s[hh * 32 + lane];
    const float et = scal[2 * hh], inv_l = scal[2 * hh + 1];
    float v[4] = {va.x, va.y, va.z, va.w};
    fwht128_warp(v, lane);  // the one inverse rotation (H = H^T = H^-1)
    const __half2 o0 = __floats2half2_rn((v[0] * sg[0] + et * tl.x) * inv_l, (v[1] * sg[1] + et * tl.y) * inv_l);
    const __half2 o1 = __floats2half2_rn((v[2] * sg[2] + et * tl.z) * inv_l, (v[3] * sg[3] + et * tl.w) * inv_l);
    *reinterpret_cast<uint2*>(out + hh * kHeadDim + 4 * lane) = make_uint2(h2_as_u32(o0), h2_as_u32(o1));
  }
  __syncwarp();
}

__device__ __forceinline__ void decode_merge_warp(const DecodeArgs& a, int b, int h, int n_rec, size_t first, int stride,
                                               bool final, float* parts, const float* tails, float* scratch,
                                               int lane) {
  switch (a.cfg.group_size) {
    case 1: decode_merge_warp_g<1>(a, b, h, n_rec, first, stride, final, parts, tails, scratch, lane); break;
    case 2: decode_merge_warp_g<2>(a, b, h, n_rec, first, stride, final, parts, tails, scratch, lane); break;
    case 3: decode_merge_warp_g<3>(a, b, h, n_rec, first, stride, final, parts, tails, scratch, lane); break;
    case 4: decode_merge_warp_g<4>(a, b, h, n_rec, first, stride, final, parts, tails, scratch, lane); break;
    case 5: decode_merge_warp_g<5>(a, b, h, n_rec, first, stride, final, parts, tails, scratch, lane); break;
    case 6: decode_merge_warp_g<6>(a, b, h, n_rec, first, stride, final, parts, tails, scratch, lane); break;
    case 7: decode_merge_warp_g<7>(a, b, h, n_rec, first, stride, final, parts, tails, scratch, lane); break;
    default: decode_merge_warp_g<8>(a, b, h, n_rec, first, stride, final, parts, tails, scratch, lane); break;
  }
}

// Where work unit u sits: sequence b, KV head h, chunk c of the S chunks of
// (b, h), ch tiles per chunk, L tokens, its first partial record at ubase.
// Decode: from the schedule (binary search of the prefix).  Serving step: a
// fixed grid of num_splits units per (b, h) over the lengths after the step;
// units with c >= S (past a short sequence's last chunk) are empty.
struct UnitLoc {
  int b, h, c, S, L, ch;
  size_t ubase;
};
template <int T>
__device__ __forceinline__ UnitLoc locate_unit(const DecodeArgs& a, int u, const int32_t* prefix,
                                               const int32_t* chunk) {
  const int nh = a.cfg.num_kv_heads;
  UnitLoc l;
  if (a.step) {
    const int sx = a.num_splits_fixed;
    l.b = u / (nh * sx);
    const int r = u - l.b * nh * sx;
    l.h = r / sx;
    l.c = r % sx;
    l.L = max(a.seq_lens[l.b], 0) + 1;
    const int f = l.L / T;
    l.ch = f > 0 ? (f + sx - 1) / sx : 1;
    l.S = f > 0 ? (f + l.ch - 1) / l.ch : 1;
    l.ubase = (static_cast<size_t>(l.b) * nh + l.h) * sx;
  } else {
    int lo = 0, hi = a.num_seqs;  // find the largest position i with nh*prefix[i] <= u
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (nh * prefix[mid] <= u) lo = mid; else hi = mid;
    }
    const int32_t* order = chunk + a.num_seqs;
    l.b = order[lo];
    l.S = prefix[lo + 1] - prefix[lo];
    const int r = u - nh * prefix[lo];
    l.h = r / l.S;
    l.c = r % l.S;
    l.L = max(a.seq_lens[l.b], 0);
    l.ch = chunk[l.b];
    l.ubase = static_cast<size_t>(nh) * prefix[lo] + static_cast<size_t>(l.h) * l.S;
  }
  return l;
}
// The first unit (chunk 0) of (sequence b, KV head h).
template <int T>
__device__ __forceinline__ UnitLoc locate_pair(const DecodeArgs& a, int b, int h, const int32_t* prefix,
                                               const int32_t* chunk) {
  const int nh = a.cfg.num_kv_heads;
  if (a.step) return locate_unit<T>(a, (b * nh + h) * a.num_splits_fixed, prefix, chunk);
  const int i = chunk[2 * a.num_seqs + b];  // rank of b in the dispatch order
  return locate_unit<T>(a, nh * prefix[i] + h * (prefix[i + 1] - prefix[i]), prefix, chunk);
}
// A merge a unit found itself last for: kind 1 = the merge group of chunks
// [first, first + n) into the record at `first`; kind 2 = the final merge of
// (b, h) over its n records (chunks or groups, `stride` apart from `ubase`).
struct PendingMerge {
  int kind = 0, b = 0, h = 0, S = 0, n = 0, stride = 1;
  size_t first = 0, ubase = 0;
  __device__ static PendingMerge group_of(int b, int h, int S, size_t ubase, size_t first, int n) {
    PendingMerge m;
    m.kind = 1; m.b = b; m.h = h; m.S = S; m.ubase = ubase; m.first = first; m.n = n; m.stride = 1;
    return m;
  }
  __device__ static PendingMerge final_of(int b, int h, int S, size_t ubase) {
    PendingMerge m;
    const int n_groups = (S + kMergeGroup - 1) / kMergeGroup;
    m.kind = 2; m.b = b; m.h = h; m.S = S; m.ubase = ubase; m.first = ubase;
    m.n = n_groups == 1 ? S : n_groups;
    m.stride = n_groups == 1 ? 1 : kMergeGroup;
    return m;
  }
};

// Arrivals that complete (sequence, KV head) at its counter: its raw-tail
// unit, its final-merge unit, and its chunk units (one merge group) or its
// merge groups.
__device__ __forceinline__ int pair_arrivals(int S) {
  const int n_groups = (S + kMergeGroup - 1) / kMergeGroup;
  return 2 + (n_groups == 1 ? S : n_groups);
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
  // per warp: two stages, at least the 8 KB the raw tail and the merge use
  // as scratch (q [8][128] and p [8][T] in fp32) once its copies have landed
  static constexpr int kWarpBytes = 2 * kStage > kTailScratch ? 2 * kStage : kTailScratch;
  // warps per CTA: 4, fewer when two stages per warp would not fit (8-bit codes)
  static constexpr int kWarps = 4 * (kWarpBytes + 16) <= 200 * 1024 ? 4 : (2 * (kWarpBytes + 16) <= 200 * 1024 ? 2 : 1);
  static constexpr int kSmem = kWarps * (kWarpBytes + 16);
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
  unsigned char* stage_base = smem + warp * Geo::kWarpBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDecWarps * Geo::kWarpBytes) + 2 * warp;
  if (lane == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncwarp();

  const int G = a.cfg.group_size, nh = a.cfg.num_kv_heads;
  const WsLayout wl = ws_layout(a.num_seqs, nh, G);
  char* ws = static_cast<char*>(a.workspace);
  int32_t* ws_i = reinterpret_cast<int32_t*>(ws);
  const int32_t* prefix = reinterpret_cast<const int32_t*>(ws + wl.prefix_off);
  const int32_t* chunk = reinterpret_cast<const int32_t*>(ws + wl.chunk_off);
  int32_t* arrivals = reinterpret_cast<int32_t*>(ws + wl.arrive_off);
  float* tails = reinterpret_cast<float*>(ws + wl.tail_off);
  float* parts = reinterpret_cast<float*>(ws + wl.part_off);
  // work items: one raw-tail unit per (sequence, KV head) first, then the
  // chunk units, then one final-merge unit per (sequence, KV head).  The tails
  // and most final merges run as bursts before and after the tile loop (their
  // code would otherwise interleave with it in the instruction cache).  Nothing
  // waits: every unit arrives at its pair's counter and whichever arrives
  // last merges (usually the final-merge unit, else a chunk still running).
  const int P = a.num_seqs * nh;
  const int UC = a.step ? a.num_seqs * nh * a.num_splits_fixed : ws_i[0];
  const int U = P + UC + P;
  int32_t* gcount = group_counters(parts, UC, G);
  const uint8_t* kpool = static_cast<const uint8_t*>(a.k_pool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.v_pool);
  const float qscale = a.softmax_scale * kLog2e / kSqrtHeadDim;
  const bool head_live = g < G;
  uint32_t phase[2] = {0u, 0u};
  bool pending[2] = {false, false};  // copies issued into the stage and not yet waited for
  bool failed = false;

  // units are handed out in order (sequence, KV head, chunk) from a queue, so
  // the chunks of one (sequence, KV head) run at about the same time and its
  // merge happens early
  while (!failed) {
    int u = 0;
    if (lane == 0) u = atomicAdd(&ws_i[1], 1);
    u = __shfl_sync(kFull, u, 0);
    if (u >= U) break;
    PendingMerge pend{};
    if (u < P || u >= P + UC) {
      // ---- raw tail of (sequence, KV head) p = (b, h): in a serving step,
      // first the step's token into tail row (L - 1) mod T; or its final-merge
      // unit, which only arrives
      const bool tail_unit = u < P;
      if (!tail_unit) u -= P + UC;
      const int b = u / nh, h = u % nh;
      const UnitLoc loc = locate_pair<T>(a, b, h, prefix, chunk);
      if (tail_unit) {
        if (a.step) step_append_warp<T>(a, b, h, loc.L, lane);
        decode_tail_warp<T>(a, b, h, loc.L % T, tails, reinterpret_cast<float*>(stage_base), lane);
        __threadfence();
      }
      __syncwarp();
      int last = 0;
      if (lane == 0) last = atomicAdd(&arrivals[u], 1) == pair_arrivals(loc.S) - 1;
      last = __shfl_sync(kFull, last, 0);
      if (last) pend = PendingMerge::final_of(b, h, loc.S, loc.ubase);
    } else {
    u -= P;
    // ---- locate the unit: sequence b, head h, chunk c of the S chunks of
    // (b, h) over L tokens (the coordinates are located again after the
    // tile loop, so that only what the loop needs stays live through it)
    UnitLoc loc = locate_unit<T>(a, u, prefix, chunk);
    if (loc.c >= loc.S) continue;  // serving step: past a short sequence's last chunk
    const int b = loc.b, h = loc.h;
    const int F = loc.L / T;
    const int t0 = loc.c * loc.ch, t1 = min(F, t0 + loc.ch);

    // block id of page `lane` (< NP) of tile `tile` of sequence b, -1 past the table
    auto tile_blk = [&](int tile) {
      const int lb = tile * NP + lane;
      return lane < NP && lb < a.max_blocks_per_seq
                 ? a.block_tables[static_cast<size_t>(b) * a.max_blocks_per_seq + lb] : -1;
    };
    // the first two tiles' block ids are read before the query, so that both
    // reads are in flight together
    const int blk0 = t0 < t1 ? tile_blk(t0) : -1;
    const int blk1 = t0 + 1 < t1 ? tile_blk(t0 + 1) : -1;

    // ---- rotated, scaled query: lane (g, t) holds channels 32t..32t+31 of head g,
    // as pairs (2i, 2i + 1) for the packed f32x2 arithmetic of the q'' fragments
    float2 qs[16];
    auto qch = [&](int i) -> float& { return (i & 1) ? qs[i >> 1].y : qs[i >> 1].x; };
    if (head_live) {
      const __half* qp = static_cast<const __half*>(a.q) +
                         ((static_cast<size_t>(b) * nh + h) * G + g) * kHeadDim + 32 * t;
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 raw = *reinterpret_cast<const uint4*>(qp + 8 * v);
        const __half2* hp = reinterpret_cast<const __half2*>(&raw);
#pragma unroll
        for (int k = 0; k < 4; ++k) qs[4 * v + k] = __half22float2(hp[k]);
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) qs[i] = make_float2(0.f, 0.f);
    }
    if (a.cfg.rotation_seed != 0) {  // q' = H D_s q
#pragma unroll
      for (int i = 0; i < 32; ++i) qch(i) *= rotation_sign(a.cfg.rotation_seed, 32 * t + i);
    }
#pragma unroll
    for (int bit = 0; bit < 5; ++bit) {  // channel bits 0..4: in-register butterflies
      const int m = 1 << bit;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (!(i & m)) {
          const float x = qch(i), y = qch(i | m);
          qch(i) = x + y;
          qch(i | m) = x - y;
        }
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {  // channel bits 5, 6: lanes with t differing in bit k
      const int m = 1 << k;
      const bool upper = t & m;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float o = __shfl_xor_sync(kFull, qch(i), m);
        qch(i) = upper ? (o - qch(i)) : (qch(i) + o);
      }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) qs[i] = __fmul2_rn(qs[i], make_float2(qscale, qscale));

    // running max; the softmax sum and the accumulator (channels 8nv + 2t,
    // 8nv + 2t + 1 in acc[nv]) as f32x2 pairs
    float m_run = -INFINITY;
    float2 l_part = make_float2(0.f, 0.f);
    float2 acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = make_float2(0.f, 0.f);

    // ---- copies of a tile's pages into stage st; lanes 0..NP-1 hold the
    // block ids of its pages and check them
    auto issue = [&](int blk, int st) {
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
    if (t0 < t1) issue(blk0, 0);
    if (t0 + 1 < t1) issue(blk1, 1);

    for (int i = t0; i < t1; ++i) {
      const int st = (i - t0) & 1;
      // T <= 64: the block ids of tile i + 2 are read now and used after this
      // tile's work; at T = 128 the extra live register costs more spills
      // than the read's latency
      constexpr bool kEarlyIds = T <= 64;
      const int blk_next = kEarlyIds && i + 2 < t1 ? tile_blk(i + 2) : -1;
      if (!pending[st]) {  // tile skipped (bad block id, already reported)
        if (i + 2 < t1) issue(kEarlyIds ? blk_next : tile_blk(i + 2), st);
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
      constexpr int kPcMax = (BK == 8 || BK == 3) ? 2 : 4;
      constexpr int kPc = NP < kPcMax ? NP : kPcMax;
      float2 sig2 = make_float2(0.f, 0.f);
      float sig = 0.f;
      float2 sc[NP][2];  // scores of tokens 8nb + 2t, 8nb + 2t + 1 of each page
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
            } else if constexpr (BK == 3) {  // 12 bytes at a 4-byte aligned offset
              const uint32_t* w = reinterpret_cast<const uint32_t*>(src);
              rec[pg][nb][0] = w[0]; rec[pg][nb][1] = w[1]; rec[pg][nb][2] = w[2];
            } else {
              const uint2 v = *reinterpret_cast<const uint2*>(src);
              rec[pg][nb][0] = v.x; rec[pg][nb][1] = v.y;
            }
          }
        // k-blocks per word: 2 (b=4), 4 (b=2), 1 (b=8); at b=3 the lane's 96
        // bits are taken as one run and every k-block extracts its 4 codes
        constexpr int kbPerWord = BK == 3 ? 8 : 8 / BK;
        constexpr int kWords = BK == 3 ? 1 : BK;
#pragma unroll
        for (int wd = 0; wd < kWords; ++wd) {
          constexpr int kPairs = BK == 3 ? 16 : 16 / BK;
          uint32_t pr[kPc][2][kPairs];
#pragma unroll
          for (int pg = 0; pg < kPc; ++pg)
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
              if constexpr (BK == 3) {
#pragma unroll
                for (int pp = 0; pp < 16; ++pp)
                  pr[pg][nb][pp] = code_pair_f16(field3(rec[pg][nb], pp), field3(rec[pg][nb], pp + 16));
              } else {
                unpack_pairs<BK>(rec[pg][nb][wd], pr[pg][nb]);
              }
            }
#pragma unroll
          for (int j = 0; j < kbPerWord; ++j) {
            const int kb = wd * kbPerWord + j;
            // pairs 2kb, 2kb+1: channels (c0, c1) and (c0+1, c1+1), c0 even
            const int c0 = pair_ch0<BK>(2 * kb), c1 = c0 + pair_gap<BK>();
            const float2 x0 = __fmul2_rn(qs[c0 >> 1], ck_pair(c0));  // channels c0, c0 + 1
            const float2 x1 = __fmul2_rn(qs[c1 >> 1], ck_pair(c1));  // channels c1, c1 + 1
            if (pc == 0) sig2 = __fadd2_rn(sig2, __fadd2_rn(x0, x1));
            // hi = fp16(x), lo = fp16(x - hi); A rows g / g + 8 take channels (c0, c1) / (c0 + 1, c1 + 1)
            const __half2 h0 = __floats2half2_rn(x0.x, x1.x), h1 = __floats2half2_rn(x0.y, x1.y);
            const float2 f0 = __half22float2(h0), f1 = __half22float2(h1);
            const float2 r0 = __fadd2_rn(x0, make_float2(-f0.x, -f1.x));
            const float2 r1 = __fadd2_rn(x1, make_float2(-f0.y, -f1.y));
            const uint32_t afr[4] = {h2_as_u32(h0), h2_as_u32(__floats2half2_rn(r0.x, r1.x)),
                                     h2_as_u32(h1), h2_as_u32(__floats2half2_rn(r0.y, r1.y))};
#pragma unroll
            for (int pg = 0; pg < kPc; ++pg)
#pragma unroll
              for (int nb = 0; nb < 2; ++nb) mma16816(sd[pg][nb], afr, pr[pg][nb][2 * j], pr[pg][nb][2 * j + 1]);
          }
        }
        if (pc == 0) {
          sig = sig2.x + sig2.y;
          sig += __shfl_xor_sync(kFull, sig, 1);
          sig += __shfl_xor_sync(kFull, sig, 2);
        }
#pragma unroll
        for (int pg = 0; pg < kPc; ++pg) {
          const unsigned char* meta = sK + (pc + pg) * Geo::kPageK + Geo::kCodesK;
#pragma unroll
          for (int nb = 0; nb < 2; ++nb) {
            // (s~, z~) of tokens 2t, 2t + 1 -> (s~, s~) and (z~, z~) pairs
            const uint2 mm = *reinterpret_cast<const uint2*>(meta + 4 * (8 * nb + 2 * t));
            const float2 sk = __half22float2(u32_as_h2(__byte_perm(mm.x, mm.y, 0x5410)));
            const float2 zk = __half22float2(u32_as_h2(__byte_perm(mm.x, mm.y, 0x7632)));
            const float2 dot = __fadd2_rn(make_float2(sd[pg][nb][0], sd[pg][nb][1]),
                                          make_float2(sd[pg][nb][2], sd[pg][nb][3]));  // hi + lo rows
            sc[pc + pg][nb] = __ffma2_rn(sk, dot, __fmul2_rn(zk, make_float2(sig, sig)));
            mt = max3f(mt, sc[pc + pg][nb].x, sc[pc + pg][nb].y);
          }
        }
      }
      mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 1));
      mt = fmaxf(mt, __shfl_xor_sync(kFull, mt, 2));
      const float m_new = fmaxf(m_run, mt);
      const float alpha = exp2f(m_run - m_new);
      m_run = m_new;
      l_part = __fmul2_rn(l_part, make_float2(alpha, alpha));

      // -- P = p * s~V as hi/lo fp16 A fragments per page; w = sum p z~V
      uint32_t pa[NP][4];
      float2 w2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int pg = 0; pg < NP; ++pg) {
        const unsigned char* meta = sV + pg * Geo::kPageV + Geo::kCodesV;
#pragma unroll
        for (int nb = 0; nb < 2; ++nb) {
          const uint2 mm = *reinterpret_cast<const uint2*>(meta + 4 * (8 * nb + 2 * t));
          const float2 sv = __half22float2(u32_as_h2(__byte_perm(mm.x, mm.y, 0x5410)));
          const float2 zv = __half22float2(u32_as_h2(__byte_perm(mm.x, mm.y, 0x7632)));
          const float2 e = __fadd2_rn(sc[pg][nb], make_float2(-m_new, -m_new));
          const float2 p = make_float2(exp2f(e.x), exp2f(e.y));
          l_part = __fadd2_rn(l_part, p);
          w2 = __ffma2_rn(p, zv, w2);
          const float2 x = __fmul2_rn(p, sv);
          const __half2 hv = __floats2half2_rn(x.x, x.y);
          const float2 hf = __half22float2(hv);
          const float2 r = __fadd2_rn(x, make_float2(-hf.x, -hf.y));
          pa[pg][2 * nb] = h2_as_u32(hv);
          pa[pg][2 * nb + 1] = h2_as_u32(__floats2half2_rn(r.x, r.y));
        }
      }
      float wsum = w2.x + w2.y;
      wsum += __shfl_xor_sync(kFull, wsum, 1);
      wsum += __shfl_xor_sync(kFull, wsum, 2);

      // -- P V: D[16 rows][8 channels] per n-block (channels 8nv..8nv+7).  Lane
      // words 2q, 2q+1 (token pairs {2t,2t+1} and {2t+8,2t+9}) hold the n-blocks
      // kPairsV*q .. kPairsV*q + kPairsV-1; a group's accumulators are folded
      // into acc' (times C~V) as soon as all pages of the tile are in.
      if constexpr (BV == 3) {
        // 3-bit V pages are a token-major bitstream: code (token p, channel c)
        // at bit 3 (128 p + c).  Lane (g, t) needs channel 8 nv + g of tokens
        // 2t, 2t+1 (B register 0) and 2t+8, 2t+9 (register 1); one read of
        // two words and a funnel shift per code.
#pragma unroll 2
        for (int nv = 0; nv < 16; ++nv) {
          const int bit = 24 * nv + 3 * g, wo = bit >> 5, sh = bit & 31;
          float dv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int pg = 0; pg < NP; ++pg) {
            const uint32_t afr[4] = {pa[pg][0], pa[pg][1], pa[pg][2], pa[pg][3]};
            const uint32_t* cw = reinterpret_cast<const uint32_t*>(sV + pg * Geo::kPageV);
            uint32_t c[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int p = 2 * t + (k & 1) + 8 * (k >> 1);
              c[k] = __funnelshift_r(cw[12 * p + wo], cw[12 * p + wo + 1], sh) & 7u;
            }
            mma16816(dv, afr, code_pair_f16(c[0], c[1]), code_pair_f16(c[2], c[3]));
          }
          const int c0 = 8 * nv + 2 * t;
          const __half2 cvh = *reinterpret_cast<const __half2*>(sV + (c0 / Geo::kCs) * Geo::kPageV + Geo::kCodesV +
                                                                64 + 2 * (c0 % Geo::kCs));
          const float2 u = __fadd2_rn(__fadd2_rn(make_float2(dv[0], dv[1]), make_float2(dv[2], dv[3])),
                                      make_float2(wsum, wsum));
          acc[nv] = __ffma2_rn(make_float2(alpha, alpha), acc[nv], __fmul2_rn(__half22float2(cvh), u));
        }
      } else {
      constexpr int kPairsV = 16 / BV;      // n-blocks per word pair
      constexpr int kGroups = 16 / kPairsV;  // word pairs per lane (4 at b=4, 2 at b=2)
      // word pairs taken together, so that kQI * kPairsV accumulators chain
      // across the pages (at least 8 MMAs between two into the same one)
      constexpr int kQI = kPairsV >= 8 ? 1 : 8 / kPairsV > kGroups ? kGroups : 8 / kPairsV;
#pragma unroll
      for (int q0 = 0; q0 < kGroups; q0 += kQI) {
        float dv[kQI][kPairsV][4];
#pragma unroll
        for (int qi = 0; qi < kQI; ++qi)
#pragma unroll
          for (int e = 0; e < kPairsV; ++e)
#pragma unroll
            for (int k = 0; k < 4; ++k) dv[qi][e][k] = 0.f;
#pragma unroll
        for (int pg = 0; pg < NP; ++pg) {
          const uint32_t afr[4] = {pa[pg][0], pa[pg][1], pa[pg][2], pa[pg][3]};
#pragma unroll
          for (int qi = 0; qi < kQI; ++qi) {
            const int q = q0 + qi;
            // words 2q and 2q+1 sit in the same 16-byte row of the lane; the whole
            // row is loaded (lanes read consecutive 16-byte rows: no bank conflict)
            const uint4 row = *reinterpret_cast<const uint4*>(sV + pg * Geo::kPageV + (((2 * q) >> 2) * 32 + lane) * 16);
            const uint32_t w0 = (q & 1) ? row.z : row.x, w1 = (q & 1) ? row.w : row.y;
            uint32_t p0[kPairsV], p1[kPairsV];
            unpack_pairs<BV>(w0, p0);
            unpack_pairs<BV>(w1, p1);
#pragma unroll
            for (int e = 0; e < kPairsV; ++e) mma16816(dv[qi][e], afr, p0[e], p1[e]);
          }
        }
#pragma unroll
        for (int qi = 0; qi < kQI; ++qi)
#pragma unroll
          for (int e = 0; e < kPairsV; ++e) {
            const int nv = kPairsV * (q0 + qi) + e;
            const int c0 = 8 * nv + 2 * t;
            const __half2 cvh = *reinterpret_cast<const __half2*>(sV + (c0 / Geo::kCs) * Geo::kPageV + Geo::kCodesV +
                                                                  64 + 2 * (c0 % Geo::kCs));
            const float2 u = __fadd2_rn(
                __fadd2_rn(make_float2(dv[qi][e][0], dv[qi][e][1]), make_float2(dv[qi][e][2], dv[qi][e][3])),
                make_float2(wsum, wsum));
            acc[nv] = __ffma2_rn(make_float2(alpha, alpha), acc[nv], __fmul2_rn(__half22float2(cvh), u));
          }
      }
      }
      __syncwarp();
      if (i + 2 < t1) issue(kEarlyIds ? blk_next : tile_blk(i + 2), st);
    }
    if (failed) break;

    // ---- partial of this unit
    float l_tot = l_part.x + l_part.y;
    l_tot += __shfl_xor_sync(kFull, l_tot, 1);
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
        *reinterpret_cast<float2*>(part + kPartAcc + c0) = acc[nv];
      }
    }
    loc = locate_unit<T>(a, u, prefix, chunk);
    // publish this unit's records; the last chunk of its group to finish
    // merges the group, the last group (or unit) of (b, h) merges the pair
    __threadfence();
    __syncwarp();
    const int n_groups = (loc.S + kMergeGroup - 1) / kMergeGroup;
    if (n_groups > 1) {
      const int j = loc.c / kMergeGroup, gsz = min(kMergeGroup, loc.S - j * kMergeGroup);
      const size_t gfirst = loc.ubase + static_cast<size_t>(j) * kMergeGroup;
      int last = 0;
      if (lane == 0) last = atomicAdd(&gcount[gfirst], 1) == gsz - 1;
      last = __shfl_sync(kFull, last, 0);
      if (last) pend = PendingMerge::group_of(loc.b, loc.h, loc.S, loc.ubase, gfirst, gsz);
    } else {
      int last = 0;
      if (lane == 0) last = atomicAdd(&arrivals[loc.b * nh + loc.h], 1) == pair_arrivals(loc.S) - 1;
      last = __shfl_sync(kFull, last, 0);
      if (last) pend = PendingMerge::final_of(loc.b, loc.h, loc.S, loc.ubase);
    }
    }
    // ---- the merges this unit completed, from one call site (inlined once):
    // a group, which may complete its (sequence, KV head); a final merge
    while (pend.kind != 0) {
      __threadfence();
      decode_merge_warp(a, pend.b, pend.h, pend.n, pend.first, pend.stride, pend.kind == 2, parts, tails,
                        reinterpret_cast<float*>(stage_base), lane);
      const int bh = pend.b * nh + pend.h;
      if (pend.kind == 1) {
        if (a.step && lane == 0) gcount[pend.first] = 0;  // the step leaves its counters at zero
        __threadfence();
        __syncwarp();
        int last = 0;
        // the pair counter counts its tail unit, its final-merge unit and its groups
        if (lane == 0) last = atomicAdd(&arrivals[bh], 1) == pair_arrivals(pend.S) - 1;
        last = __shfl_sync(kFull, last, 0);
        pend = last ? PendingMerge::final_of(pend.b, pend.h, pend.S, pend.ubase) : PendingMerge{};
      } else {
        if (a.step && lane == 0) arrivals[bh] = 0;  // the step leaves its counters at zero
        pend = PendingMerge{};
      }
    }
  }
  if (failed) {  // let copies already in flight land before the CTA's shared memory is released
    for (int st = 0; st < 2; ++st)
      if (pending[st]) (void)mbar_wait_bounded(&bars[st], phase[st]);
  }
  if (a.step) {
    // the last CTA to finish resets the unit queue and the CTA count and
    // advances every sequence's length by the step's token
    __shared__ int s_last;
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      s_last = atomicAdd(&ws_i[2], 1) == static_cast<int>(gridDim.x) - 1;
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      for (int i = threadIdx.x; i < a.num_seqs; i += blockDim.x) a.seq_lens_rw[i] = max(a.seq_lens[i], 0) + 1;
      if (threadIdx.x == 0) {
        ws_i[1] = 0;
        ws_i[2] = 0;
      }
    }
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

int device_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <int T, int BK, int BV>
cudaError_t launch_decode_bits(const DecodeArgs& a, cudaStream_t s, int sms) {
  using Geo = DecodeGeom<T, BK, BV>;
  auto kern = decode_tiles_kernel<T, BK, BV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::kSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Geo::kWarps * 32, Geo::kSmem);
  if (e != cudaSuccess) return e;
  per_sm = std::max(per_sm, 1);
  // automatic split: units_per_sm(T) units per SM (the warps take units from
  // a queue, so short units even out the ragged last chunks), as the
  // workspace holds
  const int target = units_per_sm(T) * sms;
  decode_schedule_kernel<<<1, 1024, 0, s>>>(a.seq_lens, a.num_seqs, T, a.cfg.num_kv_heads, a.cfg.group_size,
                                            a.num_splits_fixed, target, a.workspace);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  kern<<<sms * per_sm, Geo::kWarps * 32, Geo::kSmem, s>>>(a);
  return cudaGetLastError();
}

// the fused serving step: no schedule kernel (a fixed grid of num_splits
// units per (sequence, KV head)), one launch
template <int T, int BK, int BV>
cudaError_t launch_step_bits(const DecodeArgs& a, cudaStream_t s, int sms) {
  using Geo = DecodeGeom<T, BK, BV>;
  auto kern = decode_tiles_kernel<T, BK, BV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::kSmem);
  if (e != cudaSuccess) return e;
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, Geo::kWarps * 32, Geo::kSmem);
  if (e != cudaSuccess) return e;
  kern<<<sms * std::max(per_sm, 1), Geo::kWarps * 32, Geo::kSmem, s>>>(a);
  return cudaGetLastError();
}

template <int T, template <int, int, int> class L>
cudaError_t dispatch_decode_bits(const DecodeArgs& a, cudaStream_t s, int sms) {
  const int bk = a.cfg.bits_k, bv = a.cfg.bits_v;
  if (bk == 4 && bv == 4) return L<T, 4, 4>::run(a, s, sms);
  if (bk == 4 && bv == 2) return L<T, 4, 2>::run(a, s, sms);
  if (bk == 4 && bv == 3) return L<T, 4, 3>::run(a, s, sms);
  if (bk == 2 && bv == 4) return L<T, 2, 4>::run(a, s, sms);
  if (bk == 2 && bv == 3) return L<T, 2, 3>::run(a, s, sms);
  if (bk == 3 && bv == 4) return L<T, 3, 4>::run(a, s, sms);
  if (bk == 3 && bv == 2) return L<T, 3, 2>::run(a, s, sms);
  if (bk == 3 && bv == 3) return L<T, 3, 3>::run(a, s, sms);
  if (bk == 8 && bv == 8) return L<T, 8, 8>::run(a, s, sms);
  return L<T, 2, 2>::run(a, s, sms);
}
template <int T, int BK, int BV>
struct DecodeLauncher {
  static cudaError_t run(const DecodeArgs& a, cudaStream_t s, int sms) { return launch_decode_bits<T, BK, BV>(a, s, sms); }
};
template <int T, int BK, int BV>
struct StepLauncher {
  static cudaError_t run(const DecodeArgs& a, cudaStream_t s, int sms) { return launch_step_bits<T, BK, BV>(a, s, sms); }
};

template <int T>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t s) {
  return a.step ? dispatch_decode_bits<T, StepLauncher>(a, s, device_sms())
                : dispatch_decode_bits<T, DecodeLauncher>(a, s, device_sms());
}

}  // namespace

size_t decode_workspace_bytes(const kvq_config& cfg, int num_seqs, int num_splits, int num_sms) {
  if (cfg.head_dim != kHeadDim) return generic_decode_workspace_bytes(cfg, num_seqs, num_splits, num_sms);
  const WsLayout wl = ws_layout(num_seqs, cfg.num_kv_heads, cfg.group_size);
  const size_t units = num_splits > 0
                           ? static_cast<size_t>(num_seqs) * cfg.num_kv_heads * num_splits
                           : static_cast<size_t>(units_per_sm(cfg.tile_tokens)) * num_sms +
                                 static_cast<size_t>(num_seqs) * cfg.num_kv_heads;
  return wl.part_off + units * cfg.group_size * kPartFloats * sizeof(float) + units * sizeof(int32_t);
}

cudaError_t launch_selftest_wait_decode(int32_t* dev_status, cudaStream_t s) {
  selftest_wait_decode_kernel<<<1, 1, 0, s>>>(dev_status);
  return cudaGetLastError();
}

cudaError_t launch_append_decode_step(const DecodeArgs& a, cudaStream_t s) { return launch_paged_decode(a, s); }

cudaError_t launch_paged_decode(const DecodeArgs& a, cudaStream_t s) {
  if (a.cfg.head_dim != kHeadDim) return launch_generic_decode(a, s);
  if (a.num_seqs == 0) return cudaSuccess;
  switch (a.cfg.tile_tokens) {
    case 32: return launch_decode_t<32>(a, s);
    case 64: return launch_decode_t<64>(a, s);
    default: return launch_decode_t<128>(a, s);
  }
}

}  // namespace kvq
