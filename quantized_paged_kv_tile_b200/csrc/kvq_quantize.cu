// Write path: tile quantization (prefill), token append with tile
// completion, and the pool read-back used by tests and tools.
//
// Method: axbrief.com "Huawei's KVarN boosts vLLM KV-cache capacity by 5x
// without accuracy loss", section "What differs from existing methods":
// per fixed-size token tile, Hadamard rotation along the channels, then
// Sinkhorn-like alternating variance normalization, then asymmetric RTN.
//
// One CTA of 128 threads (4 warps) quantizes one (tile, KV head, K|V):
//   load + rotate : warp per token row, lane = 4 channels, warp-shuffle FWHT
//   normalize     : channel step thread-per-channel over the tile in shared
//                   memory, token step warp-per-row with shuffle reductions,
//                   in-place IEEE divisions, exact power-of-two rescaling of
//                   (C, R) after each iteration
//   RTN + pack    : warp-per-row min/max, codes OR-ed into a shared staging
//                   copy of the pages, then 16-byte stores to the pages.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {

namespace {

constexpr int kThreads = 128;
constexpr int kMaxStageWords = kPageTokens * kHeadDim * 4 / 32;  // b = 4

template <int T>
struct QuantSmem {
  float y[T][kHeadDim + 1];
  float c[kHeadDim];
  float r[T];
  __half2 meta[T];
  uint32_t stage[T / kPageTokens][kMaxStageWords];
  const __half* rows[T];
  uint8_t* pages[T / kPageTokens];
  int bcast;
  int bad;
};

// Quantize one tile whose T row pointers and T/P page pointers the caller
// put into sm.rows / sm.pages (all valid).  Ends with __syncthreads().
template <int T>
__device__ void quantize_tile_block(QuantSmem<T>& sm, const PoolGeom g, bool is_v, int iters,
                                    float eps) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int words = kPageTokens * kHeadDim * g.bits / 32;
  for (int w = tid; w < (T / kPageTokens) * kMaxStageWords; w += kThreads)
    (&sm.stage[0][0])[w] = 0u;

  // 1. rotation: Y = X H, as (X times the +-1 matrix) / sqrt(d)
  for (int i = warp; i < T; i += 4) {
    const uint2 raw = *reinterpret_cast<const uint2*>(sm.rows[i] + 4 * lane);
    const __half2 h01 = *reinterpret_cast<const __half2*>(&raw.x);
    const __half2 h23 = *reinterpret_cast<const __half2*>(&raw.y);
    float v[4] = {__low2float(h01), __high2float(h01), __low2float(h23), __high2float(h23)};
    fwht128_warp(v, lane);
#pragma unroll
    for (int k = 0; k < 4; ++k) sm.y[i][4 * lane + k] = v[k] / kSqrtHeadDim;
  }
  sm.c[tid] = 1.0f;
  for (int i = tid; i < T; i += kThreads) sm.r[i] = 1.0f;
  __syncthreads();

  // 2. normalization
  for (int it = 0; it < iters; ++it) {
    {  // channel step: thread = channel.  Deviations are taken from the
       // column's first value, so a constant column has exactly zero std.
      const int j = tid;
      const float y0 = sm.y[0][j];
      float s = 0.f;
      for (int i = 0; i < T; ++i) s += sm.y[i][j] - y0;
      const float mean = s / static_cast<float>(T);
      float q = 0.f;
      for (int i = 0; i < T; ++i) {
        const float d = (sm.y[i][j] - y0) - mean;
        q += d * d;
      }
      const float sigma = fmaxf(sqrtf(q / static_cast<float>(T)), eps);
      for (int i = 0; i < T; ++i) sm.y[i][j] = sm.y[i][j] / sigma;
      sm.c[j] *= sigma;
    }
    __syncthreads();
    for (int i = warp; i < T; i += 4) {  // token step: warp = row, shifted by the row's first value
      float v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = sm.y[i][4 * lane + k];
      const float y0 = __shfl_sync(kFull, v[0], 0);
      const float mean =
          warp_sum(((v[0] - y0) + (v[1] - y0)) + ((v[2] - y0) + (v[3] - y0))) / static_cast<float>(kHeadDim);
      float q = 0.f;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float d = (v[k] - y0) - mean;
        q += d * d;
      }
      const float rho = fmaxf(sqrtf(warp_sum(q) / static_cast<float>(kHeadDim)), eps);
#pragma unroll
      for (int k = 0; k < 4; ++k) sm.y[i][4 * lane + k] = v[k] / rho;
      if (lane == 0) sm.r[i] *= rho;
    }
    __syncthreads();
    if (warp == 0) {  // (C, R) -> (C / 2^k, R 2^k), max C in [1, 2)
      float m = fmaxf(fmaxf(sm.c[4 * lane], sm.c[4 * lane + 1]),
                      fmaxf(sm.c[4 * lane + 2], sm.c[4 * lane + 3]));
      m = warp_max(m);
      int e;
      frexpf(m, &e);
      if (lane == 0) sm.bcast = e;
    }
    __syncthreads();
    const int e = sm.bcast;
    sm.c[tid] = ldexpf(sm.c[tid], 1 - e);
    for (int i = tid; i < T; i += kThreads) sm.r[i] = ldexpf(sm.r[i], e - 1);
    __syncthreads();
  }

  // 3. per-token asymmetric RTN and packing into the staging pages
  const int qmax = (1 << g.bits) - 1;
  for (int i = warp; i < T; i += 4) {
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = sm.y[i][4 * lane + k];
    const float z = warp_min(fminf(fminf(v[0], v[1]), fminf(v[2], v[3])));
    const float mx = warp_max(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])));
    const float s = (mx - z) / static_cast<float>(qmax);
    const int page = i / kPageTokens, p = i % kPageTokens;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int code = 0;
      if (s > 0.f) {
        const float qv = rintf((v[k] - z) / s);
        code = static_cast<int>(fminf(fmaxf(qv, 0.f), static_cast<float>(qmax)));
      }
      if (code) {
        const int bit = code_bit(4 * lane + k, p, g.bits, is_v);
        const int wd = bit >> 5, off = bit & 31;
        atomicOr(&sm.stage[page][wd], static_cast<uint32_t>(code) << off);
        if (off + g.bits > 32) atomicOr(&sm.stage[page][wd + 1], static_cast<uint32_t>(code) >> (32 - off));
      }
    }
    if (lane == 0) {
      const float rr = sm.r[i];
      sm.meta[i] = __halves2half2(__float2half_rn(s * rr), __float2half_rn(z * rr));
    }
  }
  __syncthreads();

  // 4. store codes, meta and C slices into the pages
  constexpr int kPages = T / kPageTokens;
  const int vec_per_page = words / 4;
  for (int idx = tid; idx < kPages * vec_per_page; idx += kThreads) {
    const int pg = idx / vec_per_page, vi = idx % vec_per_page;
    const uint4 w = *reinterpret_cast<const uint4*>(&sm.stage[pg][4 * vi]);
    *reinterpret_cast<uint4*>(sm.pages[pg] + 16 * vi) = w;
  }
  for (int i = tid; i < T; i += kThreads) {
    const int pg = i / kPageTokens, p = i % kPageTokens;
    *reinterpret_cast<__half2*>(sm.pages[pg] + g.meta_off + 4 * p) = sm.meta[i];
  }
  {
    const int j = tid, pg = j / g.cs_channels, o = j % g.cs_channels;
    *reinterpret_cast<__half*>(sm.pages[pg] + g.cslice_off + 2 * o) = __float2half_rn(sm.c[j]);
  }
  __syncthreads();
}

// Fill sm.pages for tile `tidx` of sequence `seq`; returns false (and
// reports) when a block id is out of range.
template <int T>
__device__ bool map_tile_pages(QuantSmem<T>& sm, const int32_t* block_tables, int mb, int num_blocks,
                               int seq, int tidx, uint8_t* pool, int num_heads, int head,
                               int page_bytes, int32_t* status) {
  constexpr int kPages = T / kPageTokens;
  if (threadIdx.x == 0) sm.bad = 0;
  __syncthreads();
  if (threadIdx.x < kPages) {
    const int lb = tidx * kPages + threadIdx.x;
    const int blk = (lb < mb) ? block_tables[static_cast<size_t>(seq) * mb + lb] : -1;
    if (blk < 0 || blk >= num_blocks) {
      sm.bad = 1;
      report_error(status, KVQ_ERR_DEVICE_BOUNDS);
      sm.pages[threadIdx.x] = nullptr;
    } else {
      sm.pages[threadIdx.x] =
          pool + (static_cast<size_t>(blk) * num_heads + head) * static_cast<size_t>(page_bytes);
    }
  }
  __syncthreads();
  return sm.bad == 0;
}

template <int T>
__global__ void __launch_bounds__(kThreads) quantize_tiles_kernel(QuantizeArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  QuantSmem<T>& sm = *reinterpret_cast<QuantSmem<T>*>(smem_raw);
  const int tile = blockIdx.x, head = blockIdx.y, kv = blockIdx.z;
  const __half* src = static_cast<const __half*>(kv ? a.src_v : a.src_k);
  if (src == nullptr) return;
  const PoolGeom g = kv ? a.gv : a.gk;
  uint8_t* pool = static_cast<uint8_t*>(kv ? a.v_pool : a.k_pool);
  const int nh = a.cfg.num_kv_heads;
  const int src_row = a.tile_desc[3 * tile], seq = a.tile_desc[3 * tile + 1],
            tidx = a.tile_desc[3 * tile + 2];
  if (src_row < 0 || src_row > a.num_rows - T || seq < 0 || seq >= a.num_seqs || tidx < 0) {
    if (threadIdx.x == 0) report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
    return;
  }
  if (!map_tile_pages<T>(sm, a.block_tables, a.max_blocks_per_seq, a.num_blocks, seq, tidx, pool, nh,
                         head, g.page_bytes, a.dev_status))
    return;
  for (int i = threadIdx.x; i < T; i += kThreads)
    sm.rows[i] = src + (static_cast<size_t>(src_row + i) * nh + head) * kHeadDim;
  __syncthreads();
  quantize_tile_block<T>(sm, g, kv != 0, a.cfg.iters, a.cfg.std_eps);
}

// One CTA per (sequence, KV head, K|V): quantize every tile the new tokens
// complete (old tail rows + new rows), then write the rest into the tail.
template <int T>
__global__ void __launch_bounds__(kThreads) append_tokens_kernel(AppendArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  QuantSmem<T>& sm = *reinterpret_cast<QuantSmem<T>*>(smem_raw);
  const int b = blockIdx.x, head = blockIdx.y, kv = blockIdx.z;
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

  for (int t = l0 / T; t < end / T; ++t) {
    if (!map_tile_pages<T>(sm, a.block_tables, a.max_blocks_per_seq, a.num_blocks, b, t, pool, nh, head,
                           g.page_bytes, a.dev_status))
      continue;
    for (int i = threadIdx.x; i < T; i += kThreads) {
      const int q = t * T + i;
      sm.rows[i] = (q < l0) ? tail_base + static_cast<size_t>(q % T) * kHeadDim
                            : src + (static_cast<size_t>(start + q - l0) * nh + head) * kHeadDim;
    }
    __syncthreads();
    quantize_tile_block<T>(sm, g, kv != 0, a.cfg.iters, a.cfg.std_eps);
  }
  // remaining tokens of the unfinished tile go to the tail (16-byte pieces)
  const int first = max(l0, (end / T) * T);
  const int count = end - first;
  for (int idx = threadIdx.x; idx < count * (kHeadDim / 8); idx += kThreads) {
    const int r = idx / (kHeadDim / 8), piece = idx % (kHeadDim / 8);
    const int q = first + r;
    const uint4 v = *reinterpret_cast<const uint4*>(
        src + (static_cast<size_t>(start + q - l0) * nh + head) * kHeadDim + 8 * piece);
    *reinterpret_cast<uint4*>(tail_base + static_cast<size_t>(q % T) * kHeadDim + 8 * piece) = v;
  }
}

// Read tiles back out of a pool: codes, meta, C, dequantized values.
template <int T>
__global__ void __launch_bounds__(kThreads) unpack_tiles_kernel(UnpackArgs a) {
  constexpr int kPages = T / kPageTokens;
  __shared__ const uint8_t* pages[kPages];
  __shared__ int bad;
  const int tile = blockIdx.x, head = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nh = a.cfg.num_kv_heads;
  const PoolGeom g = a.g;
  const bool is_v = a.is_v != 0;
  const int seq = a.tile_desc[2 * tile], tidx = a.tile_desc[2 * tile + 1];
  if (tid == 0) bad = 0;
  __syncthreads();
  if (tid < kPages) {
    const int lb = tidx * kPages + tid;
    const int blk = (seq >= 0 && seq < a.num_seqs && tidx >= 0 && lb < a.max_blocks_per_seq)
                        ? a.block_tables[static_cast<size_t>(seq) * a.max_blocks_per_seq + lb]
                        : -1;
    if (blk < 0 || blk >= a.num_blocks) {
      bad = 1;
      report_error(a.dev_status, KVQ_ERR_DEVICE_BOUNDS);
    } else {
      pages[tid] = static_cast<const uint8_t*>(a.pool) +
                   (static_cast<size_t>(blk) * nh + head) * static_cast<size_t>(g.page_bytes);
    }
  }
  __syncthreads();
  if (bad) return;
  const size_t th = static_cast<size_t>(tile) * nh + head;
  if (a.cvec) {
    const int j = tid;
    static_cast<__half*>(a.cvec)[th * kHeadDim + j] = *reinterpret_cast<const __half*>(
        pages[j / g.cs_channels] + g.cslice_off + 2 * (j % g.cs_channels));
  }
  for (int i = warp; i < T; i += 4) {
    const uint8_t* pg = pages[i / kPageTokens];
    const int p = i % kPageTokens;
    const __half2 md = *reinterpret_cast<const __half2*>(pg + g.meta_off + 4 * p);
    if (a.meta && lane == 0) static_cast<__half2*>(a.meta)[th * T + i] = md;
    const float s = __low2float(md), z = __high2float(md);
    float v[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = 4 * lane + k;
      const int code = read_code(pg, code_bit(j, p, g.bits, is_v), g.bits);
      if (a.codes) a.codes[(th * T + i) * kHeadDim + j] = static_cast<uint8_t>(code);
      const float c = __half2float(*reinterpret_cast<const __half*>(
          pages[j / g.cs_channels] + g.cslice_off + 2 * (j % g.cs_channels)));
      v[k] = (static_cast<float>(code) * s + z) * c;
      if (a.out_rot) a.out_rot[(th * T + i) * kHeadDim + j] = v[k];
    }
    if (a.out_orig) {
      fwht128_warp(v, lane);
#pragma unroll
      for (int k = 0; k < 4; ++k) a.out_orig[(th * T + i) * kHeadDim + 4 * lane + k] = v[k] / kSqrtHeadDim;
    }
  }
}

template <int T>
cudaError_t launch_quantize_t(const QuantizeArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(QuantSmem<T>);
  cudaError_t e = cudaFuncSetAttribute(quantize_tiles_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_tiles, a.cfg.num_kv_heads, 2);
  quantize_tiles_kernel<T><<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int T>
cudaError_t launch_append_t(const AppendArgs& a, cudaStream_t s) {
  const size_t smem = sizeof(QuantSmem<T>);
  cudaError_t e = cudaFuncSetAttribute(append_tokens_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  dim3 grid(a.num_seqs, a.cfg.num_kv_heads, 2);
  append_tokens_kernel<T><<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace

PoolGeom pool_geom(const kvq_config& cfg, bool is_v) {
  PoolGeom g;
  g.bits = is_v ? cfg.bits_v : cfg.bits_k;
  g.codes_bytes = kPageTokens * kHeadDim * g.bits / 8;
  g.meta_off = g.codes_bytes;
  g.cs_channels = kHeadDim * kPageTokens / cfg.tile_tokens;
  g.cslice_off = g.codes_bytes + 4 * kPageTokens;
  g.page_bytes = g.cslice_off + ((2 * g.cs_channels + 15) / 16) * 16;
  g.pages_per_tile = cfg.tile_tokens / kPageTokens;
  return g;
}

cudaError_t launch_quantize_tiles(const QuantizeArgs& a, cudaStream_t s) {
  if (a.num_tiles == 0) return cudaSuccess;
  switch (a.cfg.tile_tokens) {
    case 32: return launch_quantize_t<32>(a, s);
    case 64: return launch_quantize_t<64>(a, s);
    default: return launch_quantize_t<128>(a, s);
  }
}

cudaError_t launch_append_tokens(const AppendArgs& a, cudaStream_t s) {
  if (a.num_seqs == 0) return cudaSuccess;
  switch (a.cfg.tile_tokens) {
    case 32: return launch_append_t<32>(a, s);
    case 64: return launch_append_t<64>(a, s);
    default: return launch_append_t<128>(a, s);
  }
}

cudaError_t launch_unpack_tiles(const UnpackArgs& a, cudaStream_t s) {
  if (a.num_tiles == 0) return cudaSuccess;
  dim3 grid(a.num_tiles, a.cfg.num_kv_heads);
  switch (a.cfg.tile_tokens) {
    case 32: unpack_tiles_kernel<32><<<grid, kThreads, 0, s>>>(a); break;
    case 64: unpack_tiles_kernel<64><<<grid, kThreads, 0, s>>>(a); break;
    default: unpack_tiles_kernel<128><<<grid, kThreads, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

}  // namespace kvq
