// Read path: paged decode attention over the packed pages.
//
// The attention backend reads the compressed pages directly (aitrends.kr
// article 74976, "TL;DR"; glossary "attention backend").  Per (sequence,
// KV head) the g query heads are rotated once, q' = H q; each tile t then
// contributes, in the rotated domain,
//   score_i = s~K_i (q'' . codeK_i) + z~K_i sum_j q''_j,  q'' = q' * C~K_t
//   acc'_j += C~V_tj (sum_i p_i s~V_i codeV_ij + sum_i p_i z~V_i)
// which equals softmax over q' . K^'_i and P V^' exactly in real arithmetic.
// Tiles are split into `num_splits` chunks (split-K); the merge kernel adds
// the raw fp16 tail, combines the chunks by log-sum-exp, applies the one
// inverse rotation and writes fp16.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>

#include "kvq_device.cuh"

namespace kvq {

namespace {

constexpr int kThreads = 128;
constexpr int kPartFloats = 2 + kHeadDim;  // m, l, acc[d] per query head

template <int T>
struct DecSmem {
  float qr[kMaxGroup][kHeadDim];  // rotated query * scale * log2(e)
  float qq[kMaxGroup][kHeadDim];  // q'' = q' * C~K of the current tile
  float sc[kMaxGroup][T];         // scores, then P_i = p_i * s~V_i
  float sig[kMaxGroup];
  float m[kMaxGroup], l[kMaxGroup], alpha[kMaxGroup], w[kMaxGroup];
  float ks[T], kz[T], vs[T], vz[T];
  const uint8_t* kpg[T / kPageTokens];
  const uint8_t* vpg[T / kPageTokens];
  int bad;
};

template <int T>
__global__ void __launch_bounds__(kThreads) decode_split_kernel(DecodeArgs a) {
  __shared__ DecSmem<T> sm;
  constexpr int kPages = T / kPageTokens;
  const int sp = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.cfg.group_size, nh = a.cfg.num_kv_heads, S = a.num_splits;
  const PoolGeom gk = a.gk, gv = a.gv;
  const int L = a.seq_lens[b];
  const int F = L > 0 ? L / T : 0;
  const int chunk = (F + S - 1) / S;
  const int t0 = sp * chunk, t1 = min(F, t0 + chunk);
  float* part = static_cast<float*>(a.workspace) +
                ((static_cast<size_t>(b) * nh + h) * S + sp) * G * kPartFloats;
  if (t0 >= t1) {
    if (tid < G) {
      part[tid * kPartFloats + 0] = -INFINITY;
      part[tid * kPartFloats + 1] = 0.f;
    }
    return;
  }
  const float qscale = a.softmax_scale * kLog2e / kSqrtHeadDim;
  const __half* q = static_cast<const __half*>(a.q) + (static_cast<size_t>(b) * nh + h) * G * kHeadDim;
  for (int hh = warp; hh < G; hh += 4) {
    const uint2 raw = *reinterpret_cast<const uint2*>(q + hh * kHeadDim + 4 * lane);
    const __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
    const __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
    float v[4] = {__low2float(h01), __high2float(h01), __low2float(h23), __high2float(h23)};
    fwht128_warp(v, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) sm.qr[hh][4 * lane + k] = v[k] * qscale;
  }
  if (tid < G) {
    sm.m[tid] = -INFINITY;
    sm.l[tid] = 0.f;
  }
  float acc[kMaxGroup];
#pragma unroll
  for (int hh = 0; hh < kMaxGroup; ++hh) acc[hh] = 0.f;
  const uint8_t* kpool = static_cast<const uint8_t*>(a.k_pool);
  const uint8_t* vpool = static_cast<const uint8_t*>(a.v_pool);

  for (int t = t0; t < t1; ++t) {
    if (tid == 0) sm.bad = 0;
    __syncthreads();
    if (tid < kPages) {
      const int lb = t * kPages + tid;
      const int blk = lb < a.max_blocks_per_seq
                          ? a.block_tables[static_cast<size_t>(b) * a.max_blocks_per_seq + lb]
                          : -1;
      if (blk < 0 || blk >= a.num_blocks) {
        sm.bad = 1;
        report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
      } else {
        sm.kpg[tid] = kpool + (static_cast<size_t>(blk) * nh + h) * gk.page_bytes;
        sm.vpg[tid] = vpool + (static_cast<size_t>(blk) * nh + h) * gv.page_bytes;
      }
    }
    __syncthreads();
    if (sm.bad) continue;
    const int j = tid;
    const float ck = __half2float(*reinterpret_cast<const __half*>(sm.kpg[j / gk.cs_channels] + gk.cslice_off +
                                                                    2 * (j % gk.cs_channels)));
    const float cv = __half2float(*reinterpret_cast<const __half*>(sm.vpg[j / gv.cs_channels] + gv.cslice_off +
                                                                    2 * (j % gv.cs_channels)));
    for (int hh = 0; hh < G; ++hh) sm.qq[hh][j] = sm.qr[hh][j] * ck;
    for (int i = tid; i < T; i += kThreads) {
      const int pg = i / kPageTokens, p = i % kPageTokens;
      const __half2 km = *reinterpret_cast<const __half2*>(sm.kpg[pg] + gk.meta_off + 4 * p);
      const __half2 vm = *reinterpret_cast<const __half2*>(sm.vpg[pg] + gv.meta_off + 4 * p);
      sm.ks[i] = __low2float(km);
      sm.kz[i] = __high2float(km);
      sm.vs[i] = __low2float(vm);
      sm.vz[i] = __high2float(vm);
    }
    __syncthreads();
    for (int hh = warp; hh < G; hh += 4) {
      const float s4 = (sm.qq[hh][4 * lane] + sm.qq[hh][4 * lane + 1]) +
                       (sm.qq[hh][4 * lane + 2] + sm.qq[hh][4 * lane + 3]);
      const float s = warp_sum(s4);
      if (lane == 0) sm.sig[hh] = s;
    }
    __syncthreads();
    for (int i = tid; i < T; i += kThreads) {  // scores: thread = token
      const uint8_t* pg = sm.kpg[i / kPageTokens];
      const int p = i % kPageTokens;
      float dot[kMaxGroup];
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh) dot[hh] = 0.f;
      for (int c = 0; c < kHeadDim; ++c) {
        const float code = static_cast<float>(read_code(pg, code_bit(c, p, gk.bits, false), gk.bits));
#pragma unroll
        for (int hh = 0; hh < kMaxGroup; ++hh)
          if (hh < G) dot[hh] += sm.qq[hh][c] * code;
      }
      for (int hh = 0; hh < G; ++hh) sm.sc[hh][i] = sm.ks[i] * dot[hh] + sm.kz[i] * sm.sig[hh];
    }
    __syncthreads();
    for (int hh = warp; hh < G; hh += 4) {  // online softmax over this tile
      float mt = -INFINITY;
      for (int i = lane; i < T; i += 32) mt = fmaxf(mt, sm.sc[hh][i]);
      mt = warp_max(mt);
      const float m_old = sm.m[hh];
      const float m_new = fmaxf(m_old, mt);
      float ps = 0.f, pz = 0.f;
      for (int i = lane; i < T; i += 32) {
        const float p = exp2f(sm.sc[hh][i] - m_new);
        ps += p;
        pz += p * sm.vz[i];
        sm.sc[hh][i] = p * sm.vs[i];
      }
      ps = warp_sum(ps);
      pz = warp_sum(pz);
      if (lane == 0) {
        const float al = exp2f(m_old - m_new);
        sm.alpha[hh] = al;
        sm.l[hh] = sm.l[hh] * al + ps;
        sm.m[hh] = m_new;
        sm.w[hh] = pz;
      }
    }
    __syncthreads();
    {  // P V: thread = channel
      float u[kMaxGroup];
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh) u[hh] = 0.f;
      for (int i = 0; i < T; ++i) {
        const float code = static_cast<float>(
            read_code(sm.vpg[i / kPageTokens], code_bit(j, i % kPageTokens, gv.bits, true), gv.bits));
#pragma unroll
        for (int hh = 0; hh < kMaxGroup; ++hh)
          if (hh < G) u[hh] += sm.sc[hh][i] * code;
      }
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh)
        if (hh < G) acc[hh] = acc[hh] * sm.alpha[hh] + cv * (u[hh] + sm.w[hh]);
    }
    __syncthreads();
  }
  for (int hh = 0; hh < G; ++hh) part[hh * kPartFloats + 2 + tid] = acc[hh];
  if (tid < G) {
    part[tid * kPartFloats + 0] = sm.m[tid];
    part[tid * kPartFloats + 1] = sm.l[tid];
  }
}

template <int T>
struct MergeSmem {
  float qraw[kMaxGroup][kHeadDim];
  float sc[kMaxGroup][T];
  float fin[kMaxGroup][kHeadDim];
  float tl[kMaxGroup][kHeadDim];
  float mt[kMaxGroup], lt[kMaxGroup], big_m[kMaxGroup], inv_l[kMaxGroup], et[kMaxGroup];
};

// One CTA per (sequence, KV head): raw tail, log-sum-exp merge of the
// split partials, inverse rotation, fp16 output.
template <int T>
__global__ void __launch_bounds__(kThreads) decode_merge_kernel(DecodeArgs a) {
  __shared__ MergeSmem<T> sm;
  const int h = blockIdx.x, b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = a.cfg.group_size, nh = a.cfg.num_kv_heads, S = a.num_splits;
  const int L = max(a.seq_lens[b], 0);
  const int F = L / T, tau = L - F * T;
  const float qscale = a.softmax_scale * kLog2e;
  const __half* q = static_cast<const __half*>(a.q) + (static_cast<size_t>(b) * nh + h) * G * kHeadDim;
  const __half* kt = static_cast<const __half*>(a.k_tail) + (static_cast<size_t>(b) * nh + h) * T * kHeadDim;
  const __half* vt = static_cast<const __half*>(a.v_tail) + (static_cast<size_t>(b) * nh + h) * T * kHeadDim;
  for (int hh = 0; hh < G; ++hh) sm.qraw[hh][tid] = __half2float(q[hh * kHeadDim + tid]) * qscale;
  __syncthreads();
  for (int i = tid; i < tau; i += kThreads) {
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
  for (int hh = warp; hh < G; hh += 4) {
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
    if (lane == 0) {
      sm.mt[hh] = m;
      sm.lt[hh] = ps;
    }
  }
  __syncthreads();
  {
    float at[kMaxGroup];
#pragma unroll
    for (int hh = 0; hh < kMaxGroup; ++hh) at[hh] = 0.f;
    for (int i = 0; i < tau; ++i) {
      const float vv = __half2float(vt[i * kHeadDim + tid]);
#pragma unroll
      for (int hh = 0; hh < kMaxGroup; ++hh)
        if (hh < G) at[hh] += sm.sc[hh][i] * vv;
    }
    for (int hh = 0; hh < G; ++hh) sm.tl[hh][tid] = at[hh];
  }
  const float* parts = static_cast<const float*>(a.workspace) + (static_cast<size_t>(b) * nh + h) * S * G * kPartFloats;
  if (tid < G) {
    const int hh = tid;
    float m = sm.mt[hh];
    for (int s = 0; s < S; ++s) {
      const float* pp = parts + (static_cast<size_t>(s) * G + hh) * kPartFloats;
      if (pp[1] > 0.f) m = fmaxf(m, pp[0]);
    }
    float l = sm.lt[hh] > 0.f ? sm.lt[hh] * exp2f(sm.mt[hh] - m) : 0.f;
    for (int s = 0; s < S; ++s) {
      const float* pp = parts + (static_cast<size_t>(s) * G + hh) * kPartFloats;
      if (pp[1] > 0.f) l += pp[1] * exp2f(pp[0] - m);
    }
    sm.big_m[hh] = m;
    sm.inv_l[hh] = l > 0.f ? 1.f / l : 0.f;
    sm.et[hh] = sm.lt[hh] > 0.f ? exp2f(sm.mt[hh] - m) : 0.f;
  }
  __syncthreads();
  for (int hh = 0; hh < G; ++hh) {
    float accr = 0.f;
    for (int s = 0; s < S; ++s) {
      const float* pp = parts + (static_cast<size_t>(s) * G + hh) * kPartFloats;
      if (pp[1] > 0.f) accr += exp2f(pp[0] - sm.big_m[hh]) * pp[2 + tid];
    }
    sm.fin[hh][tid] = accr;
  }
  __syncthreads();
  __half* out = static_cast<__half*>(a.out) + (static_cast<size_t>(b) * nh + h) * G * kHeadDim;
  for (int hh = warp; hh < G; hh += 4) {
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = sm.fin[hh][4 * lane + k];
    fwht128_warp(v, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int c = 4 * lane + k;
      const float o = (v[k] / kSqrtHeadDim + sm.et[hh] * sm.tl[hh][c]) * sm.inv_l[hh];
      out[hh * kHeadDim + c] = __float2half_rn(o);
    }
  }
}

template <int T>
cudaError_t launch_decode_t(const DecodeArgs& a, cudaStream_t s) {
  dim3 g1(a.num_splits, a.cfg.num_kv_heads, a.num_seqs);
  decode_split_kernel<T><<<g1, kThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  dim3 g2(a.cfg.num_kv_heads, a.num_seqs);
  decode_merge_kernel<T><<<g2, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

size_t decode_workspace_bytes(const kvq_config& cfg, int num_seqs, int num_splits) {
  return static_cast<size_t>(num_seqs) * cfg.num_kv_heads * num_splits * cfg.group_size * kPartFloats *
         sizeof(float);
}

int decode_auto_splits(const kvq_config& cfg, int num_seqs, int num_sms) {
  const long pairs = std::max(1L, static_cast<long>(num_seqs) * cfg.num_kv_heads);
  const long want = (4L * num_sms + pairs - 1) / pairs;
  return static_cast<int>(std::min(256L, std::max(1L, want)));
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
