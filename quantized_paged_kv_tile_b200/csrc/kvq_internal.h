// Internal declarations shared by the library's translation units.
// Host-side launchers: each validates nothing (the C-ABI layer in
// kvq_api.cu has done that) and returns the cudaError_t of its launches.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/kvq.h"

namespace kvq {

constexpr int kHeadDim = 128;  // the head size of the tensor-core path
constexpr int kPageTokens = 16;
constexpr int kMaxGroup = 8;

// Layout numbers of one pool (K or V), derived from the config.
struct PoolGeom {
  int bits;            // code width
  int codes_bytes;     // P*d*b/8 (d = cfg.head_dim)
  int meta_off;        // == codes_bytes
  int cslice_off;      // codes_bytes + 64
  int page_bytes;      // one (block, head) region
  int cs_channels;     // d*P/T channels of C per page
  int pages_per_tile;  // T/P
};

PoolGeom pool_geom(const kvq_config& cfg, bool is_v);

// Quantize work: one item per (tile, head, K/V).
struct QuantizeArgs {
  kvq_config cfg;
  PoolGeom gk, gv;
  const void* src_k;
  const void* src_v;
  int num_rows;
  const int32_t* tile_desc;  // [num_tiles][3]
  int num_tiles;
  const int32_t* block_tables;
  int num_seqs;
  int max_blocks_per_seq;
  int num_blocks;
  void* k_pool;
  void* v_pool;
  int32_t* dev_status;
};
cudaError_t launch_quantize_tiles(const QuantizeArgs& a, cudaStream_t s);

struct AppendArgs {
  kvq_config cfg;
  PoolGeom gk, gv;
  const void* new_k;
  const void* new_v;
  const int32_t* cu_new;
  const int32_t* seq_lens_before;
  int num_seqs;
  int max_new_per_seq;
  const int32_t* block_tables;
  int max_blocks_per_seq;
  int num_blocks;
  void* k_pool;
  void* v_pool;
  void* k_tail;
  void* v_tail;
  int32_t* dev_status;
};
cudaError_t launch_append_tokens(const AppendArgs& a, cudaStream_t s);

struct UnpackArgs {
  kvq_config cfg;
  PoolGeom g;
  const int32_t* tile_desc;  // [num_tiles][2]
  int num_tiles;
  const int32_t* block_tables;
  int num_seqs;
  int max_blocks_per_seq;
  int num_blocks;
  const void* pool;
  int is_v;
  uint8_t* codes;
  void* meta;
  void* cvec;
  float* out_rot;
  float* out_orig;
  int32_t* dev_status;
};
cudaError_t launch_unpack_tiles(const UnpackArgs& a, cudaStream_t s);

struct DecodeArgs {
  kvq_config cfg;
  PoolGeom gk, gv;
  const void* q;
  void* out;
  const int32_t* seq_lens;
  int num_seqs;
  const int32_t* block_tables;
  int max_blocks_per_seq;
  int num_blocks;
  const void* k_pool;
  const void* v_pool;
  const void* k_tail;
  const void* v_tail;
  float softmax_scale;
  void* workspace;
  int num_splits_fixed;  // > 0: chunks per (sequence, KV head); 0: automatic
  int32_t* dev_status;
  // fused serving step (kvq_append_decode_step): seq_lens hold the lengths
  // before the step; the step's K and V rows (one token per sequence) go into
  // the tails, attention runs over one more token, and the lengths advance
  int step;
  const void* new_k;       // [B][H_kv][d] fp16
  const void* new_v;
  int32_t* seq_lens_rw;    // the same array as seq_lens, written at the end of the step
};
// Workspace bytes for a split setting on a device with num_sms SMs.
size_t decode_workspace_bytes(const kvq_config& cfg, int num_seqs, int num_splits, int num_sms);
cudaError_t launch_paged_decode(const DecodeArgs& a, cudaStream_t s);
// the fused serving step: one launch (append one token per sequence, decode,
// advance the lengths); the workspace counters must be zero on entry and are
// left zero
cudaError_t launch_append_decode_step(const DecodeArgs& a, cudaStream_t s);

struct PrefillArgs {
  kvq_config cfg;
  const void* q;             // [cu_chunk[B]][H_kv*g][d] fp16
  void* out;                 // same shape
  const void* k_new;         // [cu_chunk[B]][H_kv][d] fp16
  const void* v_new;
  const int32_t* cu_chunk;   // [B+1]
  const int32_t* ctx_lens;   // [B]
  int num_seqs;
  int max_chunk;             // host bound on chunk lengths
  int row_tiles;             // 128-row query tiles per (sequence, KV head)
  const int32_t* block_tables;
  int max_blocks_per_seq;
  int num_blocks;
  const void* k_pool;
  const void* v_pool;
  const void* k_tail;
  const void* v_tail;
  float softmax_scale;
  int num_splits;            // context splits per (sequence, KV head, row tile); 1: one fused launch
  int mode;                  // 0 fused; 1 split partials (grid units x splits); 2 combine (grid units)
  float* partials;           // workspace for splits > 1: [units][splits][128][4 + d] floats
  int32_t* dev_status;
};
int prefill_row_tiles(const kvq_config& cfg, int max_chunk);
size_t prefill_workspace_bytes(const kvq_config& cfg, int num_seqs, int max_chunk, int num_splits);
cudaError_t launch_paged_prefill(const PrefillArgs& a, cudaStream_t s);

// Head sizes 64 and 256 (kvq_generic.cu): the same calls on the CUDA cores;
// the launchers above hand configurations with head_dim != 128 to these.
cudaError_t launch_generic_quantize(const QuantizeArgs& a, cudaStream_t s);
cudaError_t launch_generic_append(const AppendArgs& a, cudaStream_t s);
cudaError_t launch_generic_decode(const DecodeArgs& a, cudaStream_t s);
cudaError_t launch_generic_unpack(const UnpackArgs& a, cudaStream_t s);
size_t generic_decode_workspace_bytes(const kvq_config& cfg, int num_seqs, int num_splits, int num_sms);
// chunked prefill at d = 64 / 256: one launch, no workspace, any num_splits
// (the context is not split); CTAs of the launch
cudaError_t launch_generic_prefill(const PrefillArgs& a, cudaStream_t s);
// the serving step at d = 64 / 256: the step's tokens into the tails and the
// lengths advanced (one launch), then the decode (split-K and merge launches)
cudaError_t launch_generic_step(const DecodeArgs& a, cudaStream_t s);
long long generic_prefill_ctas(const kvq_config& cfg, int num_seqs, int max_chunk);

// Self-tests of the bounded mbarrier waits (one per kernel file): a wait on
// a barrier nothing arrives at gives up after its limit and records
// KVQ_ERR_DEVICE_TIMEOUT in *dev_status.
cudaError_t launch_selftest_wait_quantize(int32_t* dev_status, cudaStream_t s);
cudaError_t launch_selftest_wait_decode(int32_t* dev_status, cudaStream_t s);
cudaError_t launch_selftest_wait_prefill(int32_t* dev_status, cudaStream_t s);

}  // namespace kvq
