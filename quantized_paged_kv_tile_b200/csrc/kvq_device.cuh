// Device helpers shared by the kernels: the page-format bit positions,
// device error reporting, warp reductions, the warp-wide 128-point
// Walsh-Hadamard butterfly and the unpacking of code words into fp16 MMA
// operands used by both read paths.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq_internal.h"

namespace kvq {

constexpr unsigned kFull = 0xffffffffu;

// First device-detected error wins; the work item that saw it is skipped.
__device__ __forceinline__ void report_error(int32_t* status, int code) {
  if (status) atomicCAS(reinterpret_cast<int*>(status), 0, code);
}

// Bit offset of the code of (channel c, token p of the page) inside a page's
// codes region.  K, and V at 3 bits: token-major bitstream.  V at 2 / 4
// bits: grouped so that decode lane (4*g + t) owns one contiguous run of
// 32-bit words holding channels 8n+g (n = 0..15) for the token pairs
// {2t, 2t+1} and {2t+8, 2t+9}.
__device__ __forceinline__ int code_bit(int c, int p, int bits, bool is_v) {
  if (!is_v || bits == 3) return (p * kHeadDim + c) * bits;
  const int n = c >> 3, g = c & 7;
  const int t = (p & 7) >> 1, u = p >> 3, s = p & 1;
  const int h = 16 / bits;             // code pairs per 32-bit word
  const int k = 2 * (n / h) + u;       // word index inside the lane's run
  const int e = n % h;
  const int lane = 4 * g + t;
  const int word_byte = ((k >> 2) * 32 + lane) * 16 + (k & 3) * 4;
  return word_byte * 8 + bits * (e + h * s);
}

// Read one b-bit code at `bit` from a byte array (may straddle a byte).
__device__ __forceinline__ int read_code(const uint8_t* base, int bit, int bits) {
  const int byte = bit >> 3, off = bit & 7;
  unsigned v = base[byte];
  if (off + bits > 8) v |= static_cast<unsigned>(base[byte + 1]) << 8;
  return static_cast<int>((v >> off) & ((1u << bits) - 1u));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v += __shfl_xor_sync(kFull, v, m);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, m));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int m = 16; m > 0; m >>= 1) v = fminf(v, __shfl_xor_sync(kFull, v, m));
  return v;
}

// Unnormalized Walsh-Hadamard transform of one 128-vector held by a warp,
// lane L holding channels 4L..4L+3 in v[0..3].  Natural (Sylvester) order:
// the result is sum_k x_k (-1)^popcount(j & k).  Channel bits 0-1 are
// in-register butterflies, bits 2-6 pair lanes differing in bit 0-4.
__device__ __forceinline__ void fwht128_warp(float v[4], int lane) {
  const float a0 = v[0] + v[1], a1 = v[0] - v[1];
  const float a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2;
  v[2] = a0 - a2;
  v[1] = a1 + a3;
  v[3] = a1 - a3;
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const int m = 1 << k;
    const bool upper = lane & m;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float o = __shfl_xor_sync(kFull, v[i], m);
      v[i] = upper ? (o - v[i]) : (v[i] + o);
    }
  }
}

// ---- packed codes -> fp16 MMA operands (decode and chunked prefill)
__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;  // (a & b) | c
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }

// A 32-bit word of b-bit codes -> h = 16/b fp16 pairs of exact small
// integers, pair e = (field e, field e + h).
// The fields land in fp16 mantissas under the exponent of 1024 (0x6400) and
// are rebased by one subtraction or fused multiply-add.
template <int B>
__device__ __forceinline__ void unpack_pairs(uint32_t w, uint32_t out[16 / B]) {
  const uint32_t magic = 0x64006400u;
  const __half2 k1024 = __float2half2_rn(1024.f);
  if constexpr (B == 8) {  // pair e (0..1) = (byte e, byte e+2)
    out[0] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(w, 0x00FF00FFu, magic)), k1024));
    out[1] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(w >> 8, 0x00FF00FFu, magic)), k1024));
  } else if constexpr (B == 4) {  // pair e (0..3) = (nibble e, nibble e+4)
    const uint32_t w8 = w >> 8;
    const __half2 s16 = __float2half2_rn(1.f / 16.f), o64 = __float2half2_rn(-64.f);
    out[0] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(w, 0x000F000Fu, magic)), k1024));
    out[1] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(w, 0x00F000F0u, magic)), s16, o64));
    out[2] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(w8, 0x000F000Fu, magic)), k1024));
    out[3] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(w8, 0x00F000F0u, magic)), s16, o64));
  } else {  // pair e (0..7) = (field e, field e+8)
    const uint32_t w8 = w >> 8;
    const __half2 s4 = __float2half2_rn(0.25f), o256 = __float2half2_rn(-256.f);
    const __half2 s16 = __float2half2_rn(1.f / 16.f), o64 = __float2half2_rn(-64.f);
    const __half2 s64 = __float2half2_rn(1.f / 64.f), o16 = __float2half2_rn(-16.f);
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const uint32_t x = half ? w8 : w;
      out[4 * half + 0] = h2_as_u32(__hsub2(u32_as_h2(lop3_and_or(x, 0x00030003u, magic)), k1024));
      out[4 * half + 1] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(x, 0x000C000Cu, magic)), s4, o256));
      out[4 * half + 2] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(x, 0x00300030u, magic)), s16, o64));
      out[4 * half + 3] = h2_as_u32(__hfma2(u32_as_h2(lop3_and_or(x, 0x00C000C0u, magic)), s64, o16));
    }
  }
}

// Sign s_j of channel j in the randomized rotation D_s H: -1 where the j-th
// output of SplitMix64 (Steele, Lea and Flood, OOPSLA 2014) started at state
// `seed` has its top bit set, else +1; seed 0 (the plain rotation): +1.
__device__ __forceinline__ float rotation_sign(uint32_t seed, int j) {
  if (seed == 0) return 1.f;
  uint64_t z = static_cast<uint64_t>(seed) + static_cast<uint64_t>(j + 1) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  z ^= z >> 31;
  return (z >> 63) ? -1.f : 1.f;
}

constexpr float kSqrtHeadDim = 11.313708498984761f;  // sqrt(128) rounded to fp32
constexpr float kLog2e = 1.4426950408889634f;

}  // namespace kvq
