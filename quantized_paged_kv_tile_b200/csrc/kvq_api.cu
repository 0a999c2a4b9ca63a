// C ABI of the library: argument validation on the host, then the kernel
// launchers.  See include/kvq.h for the contract of every entry point.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <mutex>
#include <string>

#include "kvq_internal.h"

namespace {

thread_local std::string g_last_error;

kvq_status fail(kvq_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return s;
}

kvq_status ok() {
  g_last_error.clear();
  return KVQ_OK;
}

kvq_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

kvq_status check_config(const kvq_config* c) {
  if (c == nullptr) return fail(KVQ_ERR_INVALID_ARG, "config is NULL");
  if (c->head_dim != 64 && c->head_dim != 128 && c->head_dim != 256)
    return fail(KVQ_ERR_UNSUPPORTED, "head_dim must be 64, 128 or 256 (got %d)", c->head_dim);
  if (c->page_tokens != kvq::kPageTokens)
    return fail(KVQ_ERR_UNSUPPORTED, "page_tokens must be 16 (got %d)", c->page_tokens);
  if (c->tile_tokens != 32 && c->tile_tokens != 64 && c->tile_tokens != 128)
    return fail(KVQ_ERR_UNSUPPORTED, "tile_tokens must be 32, 64 or 128 (got %d)", c->tile_tokens);
  if (c->num_kv_heads < 1 || c->num_kv_heads > 4096)
    return fail(KVQ_ERR_INVALID_ARG, "num_kv_heads out of range (got %d)", c->num_kv_heads);
  if (c->group_size < 1 || c->group_size > kvq::kMaxGroup)
    return fail(KVQ_ERR_UNSUPPORTED, "group_size must be 1..8 (got %d)", c->group_size);
  for (int b : {c->bits_k, c->bits_v})
    if (b != 2 && b != 3 && b != 4 && b != 8)
      return fail(KVQ_ERR_UNSUPPORTED, "bits must be 2, 3, 4 or 8 (got %d)", b);
  if ((c->bits_k == 8) != (c->bits_v == 8))
    return fail(KVQ_ERR_UNSUPPORTED, "8-bit codes are for K and V together (got %d / %d)", c->bits_k, c->bits_v);
  if (c->iters < 0 || c->iters > 64) return fail(KVQ_ERR_INVALID_ARG, "iters must be 0..64 (got %d)", c->iters);
  if (!(c->std_eps > 0.f) || !(c->std_eps < 1e30f))
    return fail(KVQ_ERR_INVALID_ARG, "std_eps must be a positive finite float");
  return KVQ_OK;
}

kvq_status check_ptr(const void* p, const char* name, bool allow_null = false) {
  if (p == nullptr) {
    if (allow_null) return KVQ_OK;
    return fail(KVQ_ERR_INVALID_ARG, "%s is NULL", name);
  }
  if (!aligned16(p)) return fail(KVQ_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return KVQ_OK;
}

#define KVQ_TRY(expr)                  \
  do {                                 \
    kvq_status _s = (expr);            \
    if (_s != KVQ_OK) return _s;       \
  } while (0)

kvq_status check_tables(const int32_t* block_tables, int max_blocks_per_seq, int num_blocks) {
  KVQ_TRY(check_ptr(block_tables, "block_tables"));
  if (max_blocks_per_seq < 1) return fail(KVQ_ERR_INVALID_ARG, "max_blocks_per_seq must be >= 1");
  if (num_blocks < 1) return fail(KVQ_ERR_INVALID_ARG, "num_blocks must be >= 1");
  return KVQ_OK;
}

}  // namespace

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CUDA: return "CUDA error";
    case KVQ_ERR_WORKSPACE: return "workspace too small";
    case KVQ_ERR_DEVICE_BOUNDS: return "device saw an out-of-range block id or row";
    case KVQ_ERR_DEVICE_TIMEOUT: return "device wait timed out";
  }
  return "unknown status";
}

const char* kvq_last_error(void) { return g_last_error.c_str(); }

const char* kvq_version(void) { return "kvq 0.1 format 1 sm_100a"; }

kvq_status kvq_get_layout(const kvq_config* cfg, kvq_layout* out) {
  KVQ_TRY(check_config(cfg));
  if (out == nullptr) return fail(KVQ_ERR_INVALID_ARG, "layout output is NULL");
  const kvq::PoolGeom gk = kvq::pool_geom(*cfg, false), gv = kvq::pool_geom(*cfg, true);
  out->page_bytes_k = gk.page_bytes;
  out->page_bytes_v = gv.page_bytes;
  out->codes_bytes_k = gk.codes_bytes;
  out->codes_bytes_v = gv.codes_bytes;
  out->cslice_off_k = gk.cslice_off;
  out->cslice_off_v = gv.cslice_off;
  out->block_stride_k = static_cast<size_t>(cfg->num_kv_heads) * gk.page_bytes;
  out->block_stride_v = static_cast<size_t>(cfg->num_kv_heads) * gv.page_bytes;
  out->tail_bytes = static_cast<size_t>(cfg->num_kv_heads) * cfg->tile_tokens * cfg->head_dim * 2;
  out->cslice_channels = gk.cs_channels;
  out->pages_per_tile = gk.pages_per_tile;
  return ok();
}

kvq_status device_sm_count(int* sms) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_status(e, "querying the SM count");
  return KVQ_OK;
}

kvq_status kvq_decode_workspace_bytes(const kvq_config* cfg, int num_seqs, int num_splits, size_t* bytes) {
  KVQ_TRY(check_config(cfg));
  if (bytes == nullptr) return fail(KVQ_ERR_INVALID_ARG, "bytes output is NULL");
  if (num_seqs < 0 || num_splits < 0) return fail(KVQ_ERR_INVALID_ARG, "negative num_seqs or num_splits");
  int sms = 0;
  if (num_splits == 0) KVQ_TRY(device_sm_count(&sms));
  *bytes = kvq::decode_workspace_bytes(*cfg, num_seqs, num_splits, sms);
  return ok();
}

kvq_status kvq_quantize_tiles(const kvq_config* cfg, const void* src_k, const void* src_v, int num_rows,
                              const int32_t* tile_desc, int num_tiles, const int32_t* block_tables, int num_seqs,
                              int max_blocks_per_seq, int num_blocks, void* k_pool, void* v_pool,
                              int32_t* dev_status, void* stream) {
  KVQ_TRY(check_config(cfg));
  if (num_tiles < 0 || num_rows < 0 || num_seqs < 0)
    return fail(KVQ_ERR_INVALID_ARG, "negative num_tiles, num_rows or num_seqs");
  if (num_tiles > 0x7fffffff / 3) return fail(KVQ_ERR_INVALID_ARG, "num_tiles too large");
  if (src_k == nullptr && src_v == nullptr) return fail(KVQ_ERR_INVALID_ARG, "src_k and src_v are both NULL");
  KVQ_TRY(check_ptr(src_k, "src_k", true));
  KVQ_TRY(check_ptr(src_v, "src_v", true));
  if (num_tiles == 0) return ok();
  KVQ_TRY(check_ptr(tile_desc, "tile_desc"));
  KVQ_TRY(check_tables(block_tables, max_blocks_per_seq, num_blocks));
  KVQ_TRY(check_ptr(k_pool, "k_pool", src_k == nullptr));
  KVQ_TRY(check_ptr(v_pool, "v_pool", src_v == nullptr));
  KVQ_TRY(check_ptr(dev_status, "dev_status", true));
  if (num_tiles > 65535 * 32768) return fail(KVQ_ERR_INVALID_ARG, "num_tiles too large");
  kvq::QuantizeArgs a{};
  a.cfg = *cfg;
  a.gk = kvq::pool_geom(*cfg, false);
  a.gv = kvq::pool_geom(*cfg, true);
  a.src_k = src_k;
  a.src_v = src_v;
  a.num_rows = num_rows;
  a.tile_desc = tile_desc;
  a.num_tiles = num_tiles;
  a.block_tables = block_tables;
  a.num_seqs = num_seqs;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.dev_status = dev_status;
  return cuda_status(kvq::launch_quantize_tiles(a, static_cast<cudaStream_t>(stream)), "kvq_quantize_tiles launch");
}

kvq_status kvq_append_tokens(const kvq_config* cfg, const void* new_k, const void* new_v, const int32_t* cu_new,
                             const int32_t* seq_lens_before, int num_seqs, int max_new_per_seq,
                             const int32_t* block_tables, int max_blocks_per_seq, int num_blocks, void* k_pool,
                             void* v_pool, void* k_tail, void* v_tail, int32_t* dev_status, void* stream) {
  KVQ_TRY(check_config(cfg));
  if (num_seqs < 0 || max_new_per_seq < 0) return fail(KVQ_ERR_INVALID_ARG, "negative num_seqs or max_new_per_seq");
  if (new_k == nullptr && new_v == nullptr) return fail(KVQ_ERR_INVALID_ARG, "new_k and new_v are both NULL");
  if (num_seqs == 0 || max_new_per_seq == 0) return ok();
  if (num_seqs > 65535) return fail(KVQ_ERR_INVALID_ARG, "num_seqs > 65535");
  KVQ_TRY(check_ptr(new_k, "new_k", true));
  KVQ_TRY(check_ptr(new_v, "new_v", true));
  KVQ_TRY(check_ptr(cu_new, "cu_new"));
  KVQ_TRY(check_ptr(seq_lens_before, "seq_lens_before"));
  KVQ_TRY(check_tables(block_tables, max_blocks_per_seq, num_blocks));
  KVQ_TRY(check_ptr(k_pool, "k_pool", new_k == nullptr));
  KVQ_TRY(check_ptr(v_pool, "v_pool", new_v == nullptr));
  KVQ_TRY(check_ptr(k_tail, "k_tail", new_k == nullptr));
  KVQ_TRY(check_ptr(v_tail, "v_tail", new_v == nullptr));
  KVQ_TRY(check_ptr(dev_status, "dev_status", true));
  kvq::AppendArgs a{};
  a.cfg = *cfg;
  a.gk = kvq::pool_geom(*cfg, false);
  a.gv = kvq::pool_geom(*cfg, true);
  a.new_k = new_k;
  a.new_v = new_v;
  a.cu_new = cu_new;
  a.seq_lens_before = seq_lens_before;
  a.num_seqs = num_seqs;
  a.max_new_per_seq = max_new_per_seq;
  a.block_tables = block_tables;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.k_tail = k_tail;
  a.v_tail = v_tail;
  a.dev_status = dev_status;
  return cuda_status(kvq::launch_append_tokens(a, static_cast<cudaStream_t>(stream)), "kvq_append_tokens launch");
}

kvq_status kvq_paged_decode_attention(const kvq_config* cfg, const void* q, void* out, const int32_t* seq_lens,
                                      int num_seqs, const int32_t* block_tables, int max_blocks_per_seq,
                                      int num_blocks, const void* k_pool, const void* v_pool, const void* k_tail,
                                      const void* v_tail, float softmax_scale, void* workspace,
                                      size_t workspace_bytes, int num_splits, int32_t* dev_status, void* stream) {
  KVQ_TRY(check_config(cfg));
  if (num_seqs < 0 || num_splits < 0) return fail(KVQ_ERR_INVALID_ARG, "negative num_seqs or num_splits");
  if (num_seqs == 0) return ok();
  if (num_seqs > 65535) return fail(KVQ_ERR_INVALID_ARG, "num_seqs > 65535");
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f))
    return fail(KVQ_ERR_INVALID_ARG, "softmax_scale must be a positive finite float");
  KVQ_TRY(check_ptr(q, "q"));
  KVQ_TRY(check_ptr(out, "out"));
  KVQ_TRY(check_ptr(seq_lens, "seq_lens"));
  KVQ_TRY(check_tables(block_tables, max_blocks_per_seq, num_blocks));
  KVQ_TRY(check_ptr(k_pool, "k_pool"));
  KVQ_TRY(check_ptr(v_pool, "v_pool"));
  KVQ_TRY(check_ptr(k_tail, "k_tail"));
  KVQ_TRY(check_ptr(v_tail, "v_tail"));
  KVQ_TRY(check_ptr(workspace, "workspace"));
  KVQ_TRY(check_ptr(dev_status, "dev_status", true));
  if (num_splits > 65535) return fail(KVQ_ERR_INVALID_ARG, "num_splits > 65535");
  // the device counts work units in 32-bit ints: (num_seqs x num_kv_heads) x (splits + 2) stays below 2^30
  if (static_cast<long long>(num_seqs) * cfg->num_kv_heads * (num_splits + 2) >= (1LL << 30))
    return fail(KVQ_ERR_INVALID_ARG, "num_seqs x num_kv_heads x num_splits too large (%d x %d x %d)", num_seqs,
                cfg->num_kv_heads, num_splits);
  int sms = 0;
  if (num_splits == 0) KVQ_TRY(device_sm_count(&sms));
  const size_t need = kvq::decode_workspace_bytes(*cfg, num_seqs, num_splits, sms);
  if (workspace_bytes < need)
    return fail(KVQ_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  kvq::DecodeArgs a{};
  a.cfg = *cfg;
  a.gk = kvq::pool_geom(*cfg, false);
  a.gv = kvq::pool_geom(*cfg, true);
  a.q = q;
  a.out = out;
  a.seq_lens = seq_lens;
  a.num_seqs = num_seqs;
  a.block_tables = block_tables;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.k_tail = k_tail;
  a.v_tail = v_tail;
  a.softmax_scale = softmax_scale;
  a.workspace = workspace;
  a.num_splits_fixed = num_splits;
  a.dev_status = dev_status;
  return cuda_status(kvq::launch_paged_decode(a, static_cast<cudaStream_t>(stream)),
                     "kvq_paged_decode_attention launch");
}

kvq_status kvq_append_decode_step(const kvq_config* cfg, const void* new_k, const void* new_v, const void* q,
                                  void* out, int32_t* seq_lens, int num_seqs, const int32_t* block_tables,
                                  int max_blocks_per_seq, int num_blocks, const void* k_pool, const void* v_pool,
                                  void* k_tail, void* v_tail, float softmax_scale, void* workspace,
                                  size_t workspace_bytes, int num_splits, int32_t* dev_status, void* stream) {
  KVQ_TRY(check_config(cfg));
  if (num_seqs < 0) return fail(KVQ_ERR_INVALID_ARG, "negative num_seqs");
  if (num_seqs == 0) return ok();
  if (num_seqs > 65535) return fail(KVQ_ERR_INVALID_ARG, "num_seqs > 65535");
  if (num_splits < 1 || num_splits > 65535)
    return fail(KVQ_ERR_INVALID_ARG, "num_splits must be 1..65535 for the serving step (got %d)", num_splits);
  if (static_cast<long long>(num_seqs) * cfg->num_kv_heads * (num_splits + 2) >= (1LL << 30))
    return fail(KVQ_ERR_INVALID_ARG, "num_seqs x num_kv_heads x num_splits too large (%d x %d x %d)", num_seqs,
                cfg->num_kv_heads, num_splits);
  if (static_cast<long long>(num_seqs) * cfg->num_kv_heads * num_splits > 0x7fffffffLL)
    return fail(KVQ_ERR_INVALID_ARG, "num_seqs x num_kv_heads x num_splits too large for one launch");
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f))
    return fail(KVQ_ERR_INVALID_ARG, "softmax_scale must be a positive finite float");
  KVQ_TRY(check_ptr(new_k, "new_k"));
  KVQ_TRY(check_ptr(new_v, "new_v"));
  KVQ_TRY(check_ptr(q, "q"));
  KVQ_TRY(check_ptr(out, "out"));
  KVQ_TRY(check_ptr(seq_lens, "seq_lens"));
  KVQ_TRY(check_tables(block_tables, max_blocks_per_seq, num_blocks));
  KVQ_TRY(check_ptr(k_pool, "k_pool"));
  KVQ_TRY(check_ptr(v_pool, "v_pool"));
  KVQ_TRY(check_ptr(k_tail, "k_tail"));
  KVQ_TRY(check_ptr(v_tail, "v_tail"));
  KVQ_TRY(check_ptr(workspace, "workspace"));
  KVQ_TRY(check_ptr(dev_status, "dev_status", true));
  const size_t need = kvq::decode_workspace_bytes(*cfg, num_seqs, num_splits, 0);
  if (workspace_bytes < need)
    return fail(KVQ_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  kvq::DecodeArgs a{};
  a.cfg = *cfg;
  a.gk = kvq::pool_geom(*cfg, false);
  a.gv = kvq::pool_geom(*cfg, true);
  a.q = q;
  a.out = out;
  a.seq_lens = seq_lens;
  a.seq_lens_rw = seq_lens;
  a.num_seqs = num_seqs;
  a.block_tables = block_tables;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.k_tail = k_tail;
  a.v_tail = v_tail;
  a.softmax_scale = softmax_scale;
  a.workspace = workspace;
  a.num_splits_fixed = num_splits;
  a.dev_status = dev_status;
  a.step = 1;
  a.new_k = new_k;
  a.new_v = new_v;
  if (cfg->head_dim != kvq::kHeadDim)  // d = 64 / 256: tail write and length update, then the decode
    return cuda_status(kvq::launch_generic_step(a, static_cast<cudaStream_t>(stream)),
                       "kvq_append_decode_step launch");
  return cuda_status(kvq::launch_append_decode_step(a, static_cast<cudaStream_t>(stream)),
                     "kvq_append_decode_step launch");
}

kvq_status kvq_prefill_workspace_bytes(const kvq_config* cfg, int num_seqs, int max_chunk_tokens, int num_splits,
                                       size_t* bytes) {
  KVQ_TRY(check_config(cfg));
  if (bytes == nullptr) return fail(KVQ_ERR_INVALID_ARG, "bytes is NULL");
  if (num_seqs < 0 || max_chunk_tokens < 0) return fail(KVQ_ERR_INVALID_ARG, "negative num_seqs or max_chunk_tokens");
  if (num_splits < 1 || num_splits > 64) return fail(KVQ_ERR_INVALID_ARG, "num_splits must be 1..64");
  // d = 64 / 256: one launch over the whole context, no workspace
  *bytes = cfg->head_dim == kvq::kHeadDim ? kvq::prefill_workspace_bytes(*cfg, num_seqs, max_chunk_tokens, num_splits)
                                          : 0;
  return ok();
}

kvq_status kvq_paged_prefill_attention(const kvq_config* cfg, const void* q, void* out, const void* k_new,
                                       const void* v_new, const int32_t* cu_chunk, const int32_t* ctx_lens,
                                       int num_seqs, int max_chunk_tokens, const int32_t* block_tables,
                                       int max_blocks_per_seq, int num_blocks, const void* k_pool,
                                       const void* v_pool, const void* k_tail, const void* v_tail,
                                       float softmax_scale, int num_splits, void* workspace,
                                       size_t workspace_bytes, int32_t* dev_status, void* stream) {
  KVQ_TRY(check_config(cfg));
  const bool generic = cfg->head_dim != kvq::kHeadDim;  // d = 64 / 256: CUDA-core kernel, context not split
  if (num_splits < 1 || num_splits > 64) return fail(KVQ_ERR_INVALID_ARG, "num_splits must be 1..64");
  if (num_seqs < 0 || max_chunk_tokens < 0) return fail(KVQ_ERR_INVALID_ARG, "negative num_seqs or max_chunk_tokens");
  if (num_seqs == 0 || max_chunk_tokens == 0) return ok();
  if (num_seqs > 65535) return fail(KVQ_ERR_INVALID_ARG, "num_seqs > 65535");
  if (max_chunk_tokens > (1 << 20)) return fail(KVQ_ERR_INVALID_ARG, "max_chunk_tokens > 2^20");
  const long long units = generic ? kvq::generic_prefill_ctas(*cfg, num_seqs, max_chunk_tokens)
                                  : static_cast<long long>(num_seqs) * cfg->num_kv_heads *
                                        kvq::prefill_row_tiles(*cfg, max_chunk_tokens) * num_splits;
  if (units > 0x7fffffffLL)
    return fail(KVQ_ERR_INVALID_ARG, "num_seqs x max_chunk_tokens x num_splits too large for one launch");
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f))
    return fail(KVQ_ERR_INVALID_ARG, "softmax_scale must be a positive finite float");
  KVQ_TRY(check_ptr(q, "q"));
  KVQ_TRY(check_ptr(out, "out"));
  KVQ_TRY(check_ptr(k_new, "k_new"));
  KVQ_TRY(check_ptr(v_new, "v_new"));
  KVQ_TRY(check_ptr(cu_chunk, "cu_chunk"));
  KVQ_TRY(check_ptr(ctx_lens, "ctx_lens"));
  KVQ_TRY(check_tables(block_tables, max_blocks_per_seq, num_blocks));
  KVQ_TRY(check_ptr(k_pool, "k_pool"));
  KVQ_TRY(check_ptr(v_pool, "v_pool"));
  KVQ_TRY(check_ptr(k_tail, "k_tail"));
  KVQ_TRY(check_ptr(v_tail, "v_tail"));
  const size_t need = generic ? 0 : kvq::prefill_workspace_bytes(*cfg, num_seqs, max_chunk_tokens, num_splits);
  KVQ_TRY(check_ptr(workspace, "workspace", need == 0));
  if (workspace_bytes < need)
    return fail(KVQ_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  KVQ_TRY(check_ptr(dev_status, "dev_status", true));
  kvq::PrefillArgs a{};
  a.cfg = *cfg;
  a.q = q;
  a.out = out;
  a.k_new = k_new;
  a.v_new = v_new;
  a.cu_chunk = cu_chunk;
  a.ctx_lens = ctx_lens;
  a.num_seqs = num_seqs;
  a.max_chunk = max_chunk_tokens;
  a.row_tiles = kvq::prefill_row_tiles(*cfg, max_chunk_tokens);
  a.block_tables = block_tables;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.k_pool = k_pool;
  a.v_pool = v_pool;
  a.k_tail = k_tail;
  a.v_tail = v_tail;
  a.softmax_scale = softmax_scale;
  a.num_splits = num_splits;
  a.partials = static_cast<float*>(workspace);
  a.dev_status = dev_status;
  if (generic)
    return cuda_status(kvq::launch_generic_prefill(a, static_cast<cudaStream_t>(stream)),
                       "kvq_paged_prefill_attention launch");
  return cuda_status(kvq::launch_paged_prefill(a, static_cast<cudaStream_t>(stream)),
                     "kvq_paged_prefill_attention launch");
}

kvq_status kvq_unpack_tiles(const kvq_config* cfg, const int32_t* tile_desc, int num_tiles,
                            const int32_t* block_tables, int num_seqs, int max_blocks_per_seq, int num_blocks,
                            const void* pool,
                            int is_v, uint8_t* codes, void* meta, void* cvec, float* out_rot, float* out_orig,
                            int32_t* dev_status, void* stream) {
  KVQ_TRY(check_config(cfg));
  if (num_tiles < 0 || num_seqs < 0) return fail(KVQ_ERR_INVALID_ARG, "negative num_tiles or num_seqs");
  if (num_tiles == 0) return ok();
  if (num_tiles > 0x7fffffff) return fail(KVQ_ERR_INVALID_ARG, "num_tiles too large");
  KVQ_TRY(check_ptr(tile_desc, "tile_desc"));
  KVQ_TRY(check_tables(block_tables, max_blocks_per_seq, num_blocks));
  KVQ_TRY(check_ptr(pool, "pool"));
  KVQ_TRY(check_ptr(codes, "codes", true));
  KVQ_TRY(check_ptr(meta, "meta", true));
  KVQ_TRY(check_ptr(cvec, "cvec", true));
  KVQ_TRY(check_ptr(out_rot, "out_rot", true));
  KVQ_TRY(check_ptr(out_orig, "out_orig", true));
  KVQ_TRY(check_ptr(dev_status, "dev_status", true));
  kvq::UnpackArgs a{};
  a.cfg = *cfg;
  a.g = kvq::pool_geom(*cfg, is_v != 0);
  a.tile_desc = tile_desc;
  a.num_tiles = num_tiles;
  a.block_tables = block_tables;
  a.num_seqs = num_seqs;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_blocks = num_blocks;
  a.pool = pool;
  a.is_v = is_v != 0;
  a.codes = codes;
  a.meta = meta;
  a.cvec = cvec;
  a.out_rot = out_rot;
  a.out_orig = out_orig;
  a.dev_status = dev_status;
  return cuda_status(kvq::launch_unpack_tiles(a, static_cast<cudaStream_t>(stream)), "kvq_unpack_tiles launch");
}

kvq_status kvq_selftest_bounded_wait(int32_t* dev_status, void* stream) {
  if (dev_status == nullptr) return fail(KVQ_ERR_INVALID_ARG, "dev_status is NULL");
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  KVQ_TRY(cuda_status(kvq::launch_selftest_wait_quantize(dev_status, s), "quantize wait self-test launch"));
  KVQ_TRY(cuda_status(kvq::launch_selftest_wait_decode(dev_status, s), "decode wait self-test launch"));
  return cuda_status(kvq::launch_selftest_wait_prefill(dev_status, s), "prefill wait self-test launch");
}

}  // extern "C"

// ------------------------------------------------------- decode, static scratch
// kvq_paged_decode_attention_static_scratch runs the same decode as
// kvq_paged_decode_attention, with its workspace taken from a fixed scratch
// array compiled into the library instead of a caller-allocated buffer.  It is
// for callers that cannot allocate device memory when they decode: a runtime
// that hands the whole device to its KV pool and weights at start-up (a later
// cudaMalloc fails or fragments that budget), a serving loop that must not take
// cudaMalloc's implicit device-wide synchronization between steps, or a plain C
// embedding that links only this library and has no device allocator of its
// own.  This entry point allocates and frees nothing: it looks up the address
// of the array once per device and passes it down.
//
// The array is one per device and shared by all callers of this entry point:
// two of its calls that overlap on a device (different streams, or threads
// without ordering between their streams) race on it and corrupt each other's
// partial results.  Order them on one stream, or with events.
//
// Nothing in the scratch has to start at zero: the schedule kernel writes the
// unit counts, prefixes and chunk sizes it and the merge later read, and every
// partial record the merge reads is written by the tile kernel of the same
// call first.  So no clearing is done.
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[KVQ_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxScratchDevices] = {};

// Device address of the current device's copy of the scratch; the first call
// per device looks it up (cudaGetSymbolAddress, with that device current).
kvq_status scratch_for_current_device(void** ptr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_status(e, "querying the current device");
  if (dev < 0 || dev >= kMaxScratchDevices)
    return fail(KVQ_ERR_UNSUPPORTED, "device %d: the static decode scratch covers devices 0..%d", dev,
                kMaxScratchDevices - 1);
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return cuda_status(e, "looking up the static decode scratch");
    if (p == nullptr) return fail(KVQ_ERR_CUDA, "the static decode scratch has no device address");
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kvq_paged_decode_attention_static_scratch(
    const kvq_config* cfg, const void* q, void* out, const int32_t* seq_lens, int num_seqs,
    const int32_t* block_tables, int max_blocks_per_seq, int num_blocks, const void* k_pool, const void* v_pool,
    const void* k_tail, const void* v_tail, float softmax_scale, int num_splits, int32_t* dev_status, void* stream) {
  KVQ_TRY(check_config(cfg));
  if (num_seqs < 0) return fail(KVQ_ERR_INVALID_ARG, "num_seqs must be >= 0 (got %d)", num_seqs);
  if (num_splits < 0 || num_splits > 65535)
    return fail(KVQ_ERR_INVALID_ARG, "num_splits must be 0..65535 (got %d)", num_splits);
  int sms = 0;
  if (num_splits == 0) KVQ_TRY(device_sm_count(&sms));
  const size_t need = kvq::decode_workspace_bytes(*cfg, num_seqs, num_splits, sms);
  if (need > KVQ_DECODE_STATIC_SCRATCH_BYTES)
    return fail(KVQ_ERR_WORKSPACE,
                "decode of %d sequences (num_splits %d) needs %zu bytes of scratch; the static scratch holds %zu: "
                "pass fewer sequences or a smaller num_splits, or use kvq_paged_decode_attention with a workspace",
                num_seqs, num_splits, need, static_cast<size_t>(KVQ_DECODE_STATIC_SCRATCH_BYTES));
  void* scratch = nullptr;
  KVQ_TRY(scratch_for_current_device(&scratch));
  return kvq_paged_decode_attention(cfg, q, out, seq_lens, num_seqs, block_tables, max_blocks_per_seq, num_blocks,
                                    k_pool, v_pool, k_tail, v_tail, softmax_scale, scratch,
                                    KVQ_DECODE_STATIC_SCRATCH_BYTES, num_splits, dev_status, stream);
}
