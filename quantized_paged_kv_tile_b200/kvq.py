"""Thin ctypes binding over ``libkvq.so`` (the C ABI in ``include/kvq.h``).

Argument marshalling only: every step of the write and read paths runs in
the library's CUDA kernels.  Tensors are PyTorch CUDA tensors (PyTorch is
used for device memory and streams); each function checks dtype, shape and
contiguity, passes ``data_ptr()`` and the current stream, and raises
``KvqError`` on a non-OK status.  There is no CPU fallback: without the
built library every call raises.
"""

from __future__ import annotations

import ctypes
import dataclasses
import os

import torch

from .build import LIB_PATH

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = 1
KVQ_ERR_UNSUPPORTED = 2
KVQ_ERR_CUDA = 3
KVQ_ERR_WORKSPACE = 4
KVQ_ERR_DEVICE_BOUNDS = 5
KVQ_ERR_DEVICE_TIMEOUT = 6

EXPORTED_SYMBOLS = (
    "kvq_get_layout", "kvq_decode_workspace_bytes", "kvq_quantize_tiles", "kvq_append_tokens",
    "kvq_paged_decode_attention", "kvq_paged_decode_attention_static_scratch", "kvq_unpack_tiles",
    "kvq_selftest_bounded_wait", "kvq_status_string", "kvq_last_error", "kvq_version",
    "kvq_prefill_workspace_bytes", "kvq_paged_prefill_attention", "kvq_append_decode_step",
)


class KvqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class _Config(ctypes.Structure):
    _fields_ = [("head_dim", ctypes.c_int), ("num_kv_heads", ctypes.c_int), ("group_size", ctypes.c_int),
                ("tile_tokens", ctypes.c_int), ("page_tokens", ctypes.c_int), ("bits_k", ctypes.c_int),
                ("bits_v", ctypes.c_int), ("iters", ctypes.c_int), ("std_eps", ctypes.c_float),
                ("rotation_seed", ctypes.c_uint32)]


class _Layout(ctypes.Structure):
    _fields_ = [("page_bytes_k", ctypes.c_size_t), ("page_bytes_v", ctypes.c_size_t),
                ("codes_bytes_k", ctypes.c_size_t), ("codes_bytes_v", ctypes.c_size_t),
                ("cslice_off_k", ctypes.c_size_t), ("cslice_off_v", ctypes.c_size_t),
                ("block_stride_k", ctypes.c_size_t), ("block_stride_v", ctypes.c_size_t),
                ("tail_bytes", ctypes.c_size_t), ("cslice_channels", ctypes.c_int),
                ("pages_per_tile", ctypes.c_int)]


@dataclasses.dataclass(frozen=True)
class Config:
    """Mirror of ``kvq_config``."""
    num_kv_heads: int
    group_size: int
    tile_tokens: int
    bits_k: int
    bits_v: int
    iters: int
    head_dim: int = 128
    page_tokens: int = 16
    std_eps: float = 1e-6
    rotation_seed: int = 0  # 0: the Hadamard rotation; else the randomized rotation D_s H

    def c(self) -> _Config:
        return _Config(self.head_dim, self.num_kv_heads, self.group_size, self.tile_tokens,
                       self.page_tokens, self.bits_k, self.bits_v, self.iters, self.std_eps,
                       self.rotation_seed & 0xFFFFFFFF)

    @property
    def num_q_heads(self) -> int:
        return self.num_kv_heads * self.group_size


_LIB = None
_vp = ctypes.c_void_p
_i32 = ctypes.c_int
_sz = ctypes.c_size_t
_f32 = ctypes.c_float
_cfgp = ctypes.POINTER(_Config)

_SIGNATURES = {
    "kvq_get_layout": [_cfgp, ctypes.POINTER(_Layout)],
    "kvq_decode_workspace_bytes": [_cfgp, _i32, _i32, ctypes.POINTER(_sz)],
    "kvq_quantize_tiles": [_cfgp, _vp, _vp, _i32, _vp, _i32, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp],
    "kvq_append_tokens": [_cfgp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp],
    "kvq_paged_decode_attention": [_cfgp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _f32, _vp,
                                   _sz, _i32, _vp, _vp],
    "kvq_append_decode_step": [_cfgp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _f32,
                               _vp, _sz, _i32, _vp, _vp],
    "kvq_paged_decode_attention_static_scratch": [_cfgp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _vp, _vp, _vp,
                                                  _vp, _f32, _i32, _vp, _vp],
    "kvq_selftest_bounded_wait": [_vp, _vp],
    "kvq_prefill_workspace_bytes": [_cfgp, _i32, _i32, _i32, ctypes.POINTER(_sz)],
    "kvq_paged_prefill_attention": [_cfgp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _i32, _i32, _vp, _vp,
                                    _vp, _vp, _f32, _i32, _vp, _sz, _vp, _vp],
    "kvq_unpack_tiles": [_cfgp, _vp, _i32, _vp, _i32, _i32, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp],
}


def library_path() -> str:
    return LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load the in-tree libkvq.so; raise if it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m quantized_paged_kv_tile_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, args in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_int
    for name in ("kvq_status_string",):
        getattr(lib, name).argtypes = [ctypes.c_int]
        getattr(lib, name).restype = ctypes.c_char_p
    for name in ("kvq_last_error", "kvq_version"):
        getattr(lib, name).argtypes = []
        getattr(lib, name).restype = ctypes.c_char_p
    _LIB = lib
    return lib


def _check(status: int, what: str) -> None:
    if status != KVQ_OK:
        lib = load_library()
        msg = lib.kvq_status_string(status).decode()
        detail = lib.kvq_last_error().decode()
        raise KvqError(status, f"{what}: {msg}: {detail}")


def version() -> str:
    return load_library().kvq_version().decode()


def get_layout(cfg: Config) -> dict:
    lay = _Layout()
    _check(load_library().kvq_get_layout(ctypes.byref(cfg.c()), ctypes.byref(lay)), "kvq_get_layout")
    return {name: getattr(lay, name) for name, _ in _Layout._fields_}


def decode_workspace_bytes(cfg: Config, num_seqs: int, num_splits: int = 0) -> int:
    out = _sz(0)
    _check(load_library().kvq_decode_workspace_bytes(ctypes.byref(cfg.c()), num_seqs, num_splits,
                                                     ctypes.byref(out)), "kvq_decode_workspace_bytes")
    return out.value


def _ptr(t, name, dtype=None, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def quantize_tiles(cfg: Config, src_k, src_v, tile_desc, block_tables, k_pool, v_pool,
                   num_blocks: int | None = None, dev_status=None, stream=None) -> None:
    """Write path (prefill): quantize the tiles listed in ``tile_desc``
    (int32 [num_tiles][3] = {src_row, seq, tile_idx}) of rows ``src_k`` /
    ``src_v`` (fp16 [num_rows][H_kv][d]) into the pools."""
    src = src_k if src_k is not None else src_v
    num_rows = src.shape[0]
    pool = k_pool if k_pool is not None else v_pool
    nb = pool.shape[0] if num_blocks is None else num_blocks
    st = load_library().kvq_quantize_tiles(
        ctypes.byref(cfg.c()), _ptr(src_k, "src_k", torch.float16), _ptr(src_v, "src_v", torch.float16),
        num_rows, _ptr(tile_desc, "tile_desc", torch.int32), tile_desc.shape[0],
        _ptr(block_tables, "block_tables", torch.int32), block_tables.shape[0], block_tables.shape[1], nb,
        _ptr(k_pool, "k_pool", torch.uint8), _ptr(v_pool, "v_pool", torch.uint8),
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _check(st, "kvq_quantize_tiles")


def append_tokens(cfg: Config, new_k, new_v, cu_new, seq_lens_before, max_new_per_seq: int, block_tables,
                  k_pool, v_pool, k_tail, v_tail, num_blocks: int | None = None, dev_status=None,
                  stream=None) -> None:
    """Write path (decode / chunked prefill): append new rows, quantizing
    every tile they complete and keeping the rest in the fp16 tails."""
    pool = k_pool if k_pool is not None else v_pool
    nb = pool.shape[0] if num_blocks is None else num_blocks
    st = load_library().kvq_append_tokens(
        ctypes.byref(cfg.c()), _ptr(new_k, "new_k", torch.float16), _ptr(new_v, "new_v", torch.float16),
        _ptr(cu_new, "cu_new", torch.int32), _ptr(seq_lens_before, "seq_lens_before", torch.int32),
        seq_lens_before.shape[0], max_new_per_seq, _ptr(block_tables, "block_tables", torch.int32),
        block_tables.shape[1], nb, _ptr(k_pool, "k_pool", torch.uint8), _ptr(v_pool, "v_pool", torch.uint8),
        _ptr(k_tail, "k_tail", torch.float16), _ptr(v_tail, "v_tail", torch.float16),
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _check(st, "kvq_append_tokens")


def paged_decode_attention(cfg: Config, q, out, seq_lens, block_tables, k_pool, v_pool, k_tail, v_tail,
                           workspace, softmax_scale: float | None = None, num_splits: int = 0,
                           num_blocks: int | None = None, dev_status=None, stream=None) -> None:
    """Read path: one decode step over the packed pages (q, out fp16
    [B][H_q][d]); ``workspace`` is a uint8 CUDA tensor of at least
    ``decode_workspace_bytes`` bytes."""
    if softmax_scale is None:
        softmax_scale = cfg.head_dim ** -0.5
    nb = k_pool.shape[0] if num_blocks is None else num_blocks
    st = load_library().kvq_paged_decode_attention(
        ctypes.byref(cfg.c()), _ptr(q, "q", torch.float16), _ptr(out, "out", torch.float16),
        _ptr(seq_lens, "seq_lens", torch.int32), seq_lens.shape[0],
        _ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1], nb,
        _ptr(k_pool, "k_pool", torch.uint8), _ptr(v_pool, "v_pool", torch.uint8),
        _ptr(k_tail, "k_tail", torch.float16), _ptr(v_tail, "v_tail", torch.float16), float(softmax_scale),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), num_splits,
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _check(st, "kvq_paged_decode_attention")


def append_decode_step(cfg: Config, new_k, new_v, q, out, seq_lens, block_tables, k_pool, v_pool, k_tail, v_tail,
                       workspace, num_splits: int, softmax_scale: float | None = None, num_blocks: int | None = None,
                       dev_status=None, stream=None) -> None:
    """One serving step in one launch: the step's token rows (new_k, new_v
    fp16 [B][H_kv][d]) into the tails, decode over the cache including them,
    ``seq_lens`` (the lengths before the step) advanced by one.  No sequence
    may complete a tile in the step.  ``workspace``: uint8, at least
    ``decode_workspace_bytes(cfg, B, num_splits)`` bytes, zero-filled before
    its first use (each call leaves its counters at zero again)."""
    if softmax_scale is None:
        softmax_scale = cfg.head_dim ** -0.5
    nb = k_pool.shape[0] if num_blocks is None else num_blocks
    st = load_library().kvq_append_decode_step(
        ctypes.byref(cfg.c()), _ptr(new_k, "new_k", torch.float16), _ptr(new_v, "new_v", torch.float16),
        _ptr(q, "q", torch.float16), _ptr(out, "out", torch.float16), _ptr(seq_lens, "seq_lens", torch.int32),
        seq_lens.shape[0], _ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1], nb,
        _ptr(k_pool, "k_pool", torch.uint8), _ptr(v_pool, "v_pool", torch.uint8),
        _ptr(k_tail, "k_tail", torch.float16), _ptr(v_tail, "v_tail", torch.float16), float(softmax_scale),
        _ptr(workspace, "workspace", torch.uint8), workspace.numel(), num_splits,
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _check(st, "kvq_append_decode_step")


def step_splits(cfg: Config, num_seqs: int, num_sms: int) -> int:
    """Chunks per (sequence, KV head) for the fused serving step: about 32
    work units per SM (the granularity the automatic decode split uses), at
    least one per (sequence, KV head)."""
    pairs = max(1, num_seqs * cfg.num_kv_heads)
    return min(65535, max(1, -(-32 * num_sms // pairs)))


def prefill_workspace_bytes(cfg: Config, num_seqs: int, max_chunk_tokens: int, num_splits: int) -> int:
    out = _sz(0)
    _check(load_library().kvq_prefill_workspace_bytes(ctypes.byref(cfg.c()), num_seqs, max_chunk_tokens, num_splits,
                                                      ctypes.byref(out)), "kvq_prefill_workspace_bytes")
    return out.value


def prefill_splits(cfg: Config, num_seqs: int, max_chunk_tokens: int, max_context_tokens: int,
                   num_sms: int) -> int:
    """A context split count for kvq_paged_prefill_attention: the smallest S
    (each split keeping at least 16 tiles) whose CTA count fills its last wave
    to 99%, else the best fill found."""
    units = num_seqs * cfg.num_kv_heads * -(-max_chunk_tokens * cfg.group_size // 128)
    if units == 0:
        return 1
    tiles = max_context_tokens // cfg.tile_tokens
    best, best_fill = 1, 0.0
    for s in range(1, 17):
        if s > 1 and tiles // s < 16:
            break
        n = units * s
        fill = n / (-(-n // num_sms) * num_sms)
        if fill >= 0.99:
            return s
        if fill > best_fill + 1e-9:
            best, best_fill = s, fill
    return best


def paged_prefill_attention(cfg: Config, q, out, k_new, v_new, cu_chunk, ctx_lens, max_chunk_tokens: int,
                            block_tables, k_pool, v_pool, k_tail, v_tail, num_splits: int = 1, workspace=None,
                            softmax_scale: float | None = None, num_blocks: int | None = None, dev_status=None,
                            stream=None) -> None:
    """Read path, chunked prefill: chunk rows (q, out fp16 [N][H_q][d];
    k_new, v_new fp16 [N][H_kv][d], N = cu_chunk[-1]) attend to the cached
    context of their sequence and causally to their own chunk.  With
    ``num_splits`` > 1, ``workspace`` is a uint8 CUDA tensor of at least
    ``prefill_workspace_bytes`` bytes."""
    if softmax_scale is None:
        softmax_scale = cfg.head_dim ** -0.5
    nb = k_pool.shape[0] if num_blocks is None else num_blocks
    st = load_library().kvq_paged_prefill_attention(
        ctypes.byref(cfg.c()), _ptr(q, "q", torch.float16), _ptr(out, "out", torch.float16),
        _ptr(k_new, "k_new", torch.float16), _ptr(v_new, "v_new", torch.float16),
        _ptr(cu_chunk, "cu_chunk", torch.int32), _ptr(ctx_lens, "ctx_lens", torch.int32), ctx_lens.shape[0],
        int(max_chunk_tokens), _ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1], nb,
        _ptr(k_pool, "k_pool", torch.uint8), _ptr(v_pool, "v_pool", torch.uint8),
        _ptr(k_tail, "k_tail", torch.float16), _ptr(v_tail, "v_tail", torch.float16), float(softmax_scale),
        int(num_splits), _ptr(workspace, "workspace", torch.uint8), 0 if workspace is None else workspace.numel(),
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _check(st, "kvq_paged_prefill_attention")


# bytes of the library's static decode scratch (one per device)
DECODE_STATIC_SCRATCH_BYTES = 32 << 20


def paged_decode_attention_static_scratch(cfg: Config, q, out, seq_lens, block_tables, k_pool, v_pool, k_tail,
                                          v_tail, softmax_scale: float | None = None, num_splits: int = 0,
                                          num_blocks: int | None = None, dev_status=None, stream=None) -> None:
    """``paged_decode_attention`` on the library's static per-device scratch
    instead of a workspace: allocates nothing.  Calls that overlap on one
    device race on that scratch; the first call per device should come before
    any stream capture."""
    if softmax_scale is None:
        softmax_scale = cfg.head_dim ** -0.5
    nb = k_pool.shape[0] if num_blocks is None else num_blocks
    st = load_library().kvq_paged_decode_attention_static_scratch(
        ctypes.byref(cfg.c()), _ptr(q, "q", torch.float16), _ptr(out, "out", torch.float16),
        _ptr(seq_lens, "seq_lens", torch.int32), seq_lens.shape[0],
        _ptr(block_tables, "block_tables", torch.int32), block_tables.shape[1], nb,
        _ptr(k_pool, "k_pool", torch.uint8), _ptr(v_pool, "v_pool", torch.uint8),
        _ptr(k_tail, "k_tail", torch.float16), _ptr(v_tail, "v_tail", torch.float16), float(softmax_scale),
        num_splits, _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _check(st, "kvq_paged_decode_attention_static_scratch")


def selftest_bounded_wait(dev_status, stream=None) -> None:
    """Run the device-side bounded-wait self-test (about 6 s): afterwards
    ``dev_status`` holds KVQ_ERR_DEVICE_TIMEOUT."""
    st = load_library().kvq_selftest_bounded_wait(_ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _check(st, "kvq_selftest_bounded_wait")


def unpack_tiles(cfg: Config, tile_desc, block_tables, pool, is_v: bool, codes=None, meta=None, cvec=None,
                 out_rot=None, out_orig=None, num_blocks: int | None = None, dev_status=None,
                 stream=None) -> None:
    """Read tiles ({seq, tile_idx} rows of ``tile_desc``) back out of a pool."""
    nb = pool.shape[0] if num_blocks is None else num_blocks
    st = load_library().kvq_unpack_tiles(
        ctypes.byref(cfg.c()), _ptr(tile_desc, "tile_desc", torch.int32), tile_desc.shape[0],
        _ptr(block_tables, "block_tables", torch.int32), block_tables.shape[0], block_tables.shape[1], nb,
        _ptr(pool, "pool", torch.uint8), int(bool(is_v)), _ptr(codes, "codes", torch.uint8),
        _ptr(meta, "meta", torch.float16), _ptr(cvec, "cvec", torch.float16),
        _ptr(out_rot, "out_rot", torch.float32), _ptr(out_orig, "out_orig", torch.float32),
        _ptr(dev_status, "dev_status", torch.int32), _stream(stream))
    _check(st, "kvq_unpack_tiles")
