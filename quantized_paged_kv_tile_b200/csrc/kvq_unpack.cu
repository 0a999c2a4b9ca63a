// Pool read-back for tests and tools (kvq_unpack_tiles): codes, fp16
// metadata, C vectors and dequantized tiles, X^' = (code s~ + z~) C~ in the
// rotated domain and X^ = X^' H in the original one.  Also the page geometry
// shared by all launchers.
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kvq_device.cuh"

namespace kvq {

namespace {

constexpr int kThreads = 128;

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
      for (int k = 0; k < 4; ++k)  // X^ = X^' H D_s
        a.out_orig[(th * T + i) * kHeadDim + 4 * lane + k] =
            v[k] / kSqrtHeadDim * rotation_sign(a.cfg.rotation_seed, 4 * lane + k);
    }
  }
}

}  // namespace

PoolGeom pool_geom(const kvq_config& cfg, bool is_v) {
  PoolGeom g;
  g.bits = is_v ? cfg.bits_v : cfg.bits_k;
  g.codes_bytes = kPageTokens * cfg.head_dim * g.bits / 8;
  g.meta_off = g.codes_bytes;
  g.cs_channels = cfg.head_dim * kPageTokens / cfg.tile_tokens;
  g.cslice_off = g.codes_bytes + 4 * kPageTokens;
  g.page_bytes = g.cslice_off + ((2 * g.cs_channels + 15) / 16) * 16;
  g.pages_per_tile = cfg.tile_tokens / kPageTokens;
  return g;
}

cudaError_t launch_unpack_tiles(const UnpackArgs& a, cudaStream_t s) {
  if (a.cfg.head_dim != kHeadDim) return launch_generic_unpack(a, s);
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
