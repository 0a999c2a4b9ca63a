"""Host-side bookkeeping of a quantized paged KV cache (one attention layer).

``PagedKVCache`` owns the device buffers the C ABI works on (K/V page
pools, fp16 tails, block tables, sequence lengths, decode workspace) and
turns user-level operations into the three library calls:
  prefill(rows)  -> kvq_quantize_tiles for every full tile, then
                    kvq_append_tokens for the unfinished last tile
  append(rows)   -> kvq_append_tokens (quantizes tiles as they fill)
  decode(q)      -> kvq_paged_decode_attention
  prefill_chunk(q, rows) -> kvq_paged_prefill_attention over the cache and
                    the chunk, then kvq_append_tokens of the chunk
All arithmetic runs in the library's kernels; this module only sizes and
indexes buffers (PyTorch provides the memory and the stream).
"""

from __future__ import annotations

import math

import contextlib

import numpy as np
import torch

from . import kvq


@contextlib.contextmanager
def _on_stream(stream):
    """Run the enclosed calls on ``stream`` (a torch.cuda.Stream, or None for
    the current stream): temporaries made inside are allocated and copied on
    it, so the caching allocator never hands their memory to other work while
    the stream's kernels still read it."""
    if stream is None:
        yield
    else:
        with torch.cuda.stream(stream):
            yield


def _in_use(buf):
    """Mark a long-lived buffer as used by the current stream (it may have
    been allocated on another), so that freeing it later waits for this use."""
    if buf is not None and buf.is_cuda:
        buf.record_stream(torch.cuda.current_stream(buf.device))


class PagedKVCache:
    def __init__(self, cfg: kvq.Config, num_seqs: int, max_tokens_per_seq: int, device="cuda",
                 block_table: np.ndarray | None = None, num_splits: int = 0):
        self.cfg = cfg
        self.num_seqs = num_seqs
        self.device = torch.device(device)
        self.layout = kvq.get_layout(cfg)
        self.blocks_per_seq = math.ceil(max_tokens_per_seq / cfg.page_tokens)
        if block_table is None:
            block_table = np.arange(num_seqs * self.blocks_per_seq, dtype=np.int32).reshape(num_seqs, -1)
        if block_table.shape != (num_seqs, self.blocks_per_seq):
            raise ValueError(f"block table shape {block_table.shape} != {(num_seqs, self.blocks_per_seq)}")
        self.num_blocks = int(block_table.max()) + 1
        self.block_tables = torch.from_numpy(np.ascontiguousarray(block_table, dtype=np.int32)).to(self.device)
        h = cfg.num_kv_heads
        self.k_pool = torch.zeros((self.num_blocks, h, self.layout["page_bytes_k"]), dtype=torch.uint8,
                                  device=self.device)
        self.v_pool = torch.zeros((self.num_blocks, h, self.layout["page_bytes_v"]), dtype=torch.uint8,
                                  device=self.device)
        tail_shape = (num_seqs, h, cfg.tile_tokens, cfg.head_dim)
        self.k_tail = torch.zeros(tail_shape, dtype=torch.float16, device=self.device)
        self.v_tail = torch.zeros(tail_shape, dtype=torch.float16, device=self.device)
        self.seq_lens = torch.zeros(num_seqs, dtype=torch.int32, device=self.device)
        self.host_lens = np.zeros(num_seqs, dtype=np.int64)
        self.num_splits = num_splits
        self.workspace = torch.empty(kvq.decode_workspace_bytes(cfg, num_seqs, num_splits), dtype=torch.uint8,
                                     device=self.device)
        self.prefill_workspace = None  # grown on demand by prefill_chunk when it splits contexts
        self.dev_status = torch.zeros(1, dtype=torch.int32, device=self.device)

    # ------------------------------------------------------------------ write
    def prefill_tile_desc(self, lens) -> np.ndarray:
        """{src_row, seq, tile_idx} for every full tile of packed rows with
        per-sequence lengths ``lens`` (rows of seq s start at sum(lens[:s]))."""
        t = self.cfg.tile_tokens
        starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
        desc = [(starts[s] + i * t, s, i) for s in range(len(lens)) for i in range(int(lens[s]) // t)]
        return np.asarray(desc, dtype=np.int32).reshape(-1, 3)

    def prefill(self, rows_k: torch.Tensor, rows_v: torch.Tensor, lens, stream=None) -> None:
        """Load an empty cache with packed rows [sum(lens)][H_kv][d]."""
        lens = np.asarray(lens, dtype=np.int64)
        if np.any(self.host_lens):
            raise RuntimeError("prefill expects an empty cache")
        with _on_stream(stream):
            desc = torch.from_numpy(self.prefill_tile_desc(lens)).to(self.device)
            kvq.quantize_tiles(self.cfg, rows_k, rows_v, desc, self.block_tables, self.k_pool, self.v_pool,
                               num_blocks=self.num_blocks, dev_status=self.dev_status)
            t = self.cfg.tile_tokens
            full = (lens // t) * t
            rest = lens - full
            if rest.any():
                starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
                idx = np.concatenate([np.arange(starts[s] + full[s], starts[s] + lens[s]) for s in range(len(lens))])
                idx_t = torch.from_numpy(idx).to(self.device)
                self._append(rows_k.index_select(0, idx_t), rows_v.index_select(0, idx_t), full, rest)
            self.host_lens = lens.copy()
            self.seq_lens.copy_(torch.from_numpy(lens.astype(np.int32)))

    def _append(self, new_k, new_v, before, counts) -> None:
        # runs on the current stream (callers enter _on_stream first)
        cu = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        kvq.append_tokens(self.cfg, new_k, new_v, torch.from_numpy(cu).to(self.device),
                          torch.from_numpy(np.asarray(before, dtype=np.int32)).to(self.device),
                          int(np.max(counts)), self.block_tables, self.k_pool, self.v_pool, self.k_tail,
                          self.v_tail, num_blocks=self.num_blocks, dev_status=self.dev_status)

    def append(self, new_k: torch.Tensor, new_v: torch.Tensor, counts=None, stream=None) -> None:
        """Append packed rows (``counts`` per sequence, default one each)."""
        if counts is None:
            counts = np.ones(self.num_seqs, dtype=np.int64)
        counts = np.asarray(counts, dtype=np.int64)
        if np.any(self.host_lens + counts > self.blocks_per_seq * self.cfg.page_tokens):
            raise ValueError("append past the allocated pages")
        with _on_stream(stream):
            self._append(new_k, new_v, self.host_lens, counts)
            self.host_lens = self.host_lens + counts
            self.seq_lens.copy_(torch.from_numpy(self.host_lens.astype(np.int32)))

    # ------------------------------------------------------------------- read
    def decode(self, q: torch.Tensor, out: torch.Tensor | None = None, num_splits: int | None = None,
               stream=None) -> torch.Tensor:
        """One decode step: q fp16 [B][H_q][d] -> out fp16 [B][H_q][d]."""
        splits = self.num_splits if num_splits is None else num_splits
        with _on_stream(stream):
            if out is None:
                out = torch.empty_like(q)
            ws = self.workspace
            need = kvq.decode_workspace_bytes(self.cfg, self.num_seqs, splits)
            if ws.numel() < need:
                ws = torch.empty(need, dtype=torch.uint8, device=self.device)  # freed after this call's work
            else:
                _in_use(ws)
            kvq.paged_decode_attention(self.cfg, q, out, self.seq_lens, self.block_tables, self.k_pool,
                                       self.v_pool, self.k_tail, self.v_tail, ws, num_splits=splits,
                                       num_blocks=self.num_blocks, dev_status=self.dev_status)
        return out

    def prefill_chunk(self, q: torch.Tensor, new_k: torch.Tensor, new_v: torch.Tensor, counts,
                      out: torch.Tensor | None = None, append: bool = True, num_splits: int | None = None,
                      stream=None) -> torch.Tensor:
        """Chunked prefill: packed chunk rows (``counts`` tokens per sequence;
        q fp16 [N][H_q][d], new_k / new_v fp16 [N][H_kv][d]) attend to the
        cached context and causally to their own chunk; then (``append``) the
        chunk joins the cache.  ``num_splits`` (default: chosen from the
        context lengths and the SM count) splits long contexts over more
        CTAs.  Returns out fp16 [N][H_q][d]."""
        counts = np.asarray(counts, dtype=np.int64)
        if counts.shape != (self.num_seqs,) or np.any(counts < 0):
            raise ValueError("counts: one non-negative chunk length per sequence")
        if append and np.any(self.host_lens + counts > self.blocks_per_seq * self.cfg.page_tokens):
            raise ValueError("append past the allocated pages")
        max_chunk = int(counts.max()) if counts.size else 0
        if num_splits is None:
            num_splits = 1
            if self.device.type == "cuda":  # (anything else is refused by the binding below)
                sms = torch.cuda.get_device_properties(self.device).multi_processor_count
                num_splits = kvq.prefill_splits(self.cfg, self.num_seqs, max_chunk, int(self.host_lens.max()), sms)
        need = kvq.prefill_workspace_bytes(self.cfg, self.num_seqs, max_chunk, num_splits)
        with _on_stream(stream):
            if out is None:
                out = torch.empty_like(q)
            cu = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).to(self.device)
            ws = None
            if need > 0:
                if self.prefill_workspace is None or self.prefill_workspace.numel() < need:
                    # the old buffer (if any) may still be read by earlier work on
                    # another stream: it was marked in use there when it was used
                    self.prefill_workspace = torch.empty(need, dtype=torch.uint8, device=self.device)
                ws = self.prefill_workspace
                _in_use(ws)
            kvq.paged_prefill_attention(self.cfg, q, out, new_k, new_v, cu, self.seq_lens, max_chunk,
                                        self.block_tables, self.k_pool, self.v_pool, self.k_tail, self.v_tail,
                                        num_splits=num_splits, workspace=ws, num_blocks=self.num_blocks,
                                        dev_status=self.dev_status)
            if append and max_chunk > 0:
                self._append(new_k, new_v, self.host_lens, counts)
                self.host_lens = self.host_lens + counts
                self.seq_lens.copy_(torch.from_numpy(self.host_lens.astype(np.int32)))
        return out

    def status(self) -> int:
        """Device status word (0 = no device-detected error); synchronizes."""
        return int(self.dev_status.item())

    def bytes_per_token_head(self) -> float:
        """Stored bytes per (token, KV head) for K+V, pages only."""
        p = self.cfg.page_tokens
        return (self.layout["page_bytes_k"] + self.layout["page_bytes_v"]) / p


class DecodeStepGraph:
    """One serving step of a ``PagedKVCache`` -- append one token per sequence,
    then decode -- captured once in a CUDA graph and replayed.

    Stage the step's rows in ``new_k`` / ``new_v`` ([B][H_kv][d] fp16) and its
    queries in ``q`` ([B][H_q][d] fp16), call ``replay()``, read ``out``.  The
    sequence lengths advance on the device inside the graph (the append reads
    them as the lengths before the step, then they grow by one); the host
    tracks them to refuse a step past the allocated pages.  The first decode
    and append calls happen eagerly before capture.

    ``fused=True``: steps in which no sequence completes a tile replay a graph
    of one launch (kvq_append_decode_step: the token into the tails, the
    decode, the lengths advanced); steps that complete a tile replay the
    append + decode graph (the completed tile has to be quantized first).
    Both use the same split count, so the outputs are those of the unfused
    step bit for bit.
    """

    def __init__(self, cache: PagedKVCache, num_splits: int | None = None, fused: bool = False):
        self.cache = cache
        cfg, b, dev = cache.cfg, cache.num_seqs, cache.device
        self.fused = fused
        if fused and num_splits is None:
            num_splits = kvq.step_splits(cfg, b, torch.cuda.get_device_properties(dev).multi_processor_count)
        self.num_splits = cache.num_splits if num_splits is None else num_splits
        self.new_k = torch.zeros((b, cfg.num_kv_heads, cfg.head_dim), dtype=torch.float16, device=dev)
        self.new_v = torch.zeros_like(self.new_k)
        self.q = torch.zeros((b, cfg.num_q_heads, cfg.head_dim), dtype=torch.float16, device=dev)
        self.out = torch.empty_like(self.q)
        self._cu = torch.arange(b + 1, dtype=torch.int32, device=dev)
        need = kvq.decode_workspace_bytes(cfg, b, self.num_splits)
        if cache.workspace.numel() < need:
            cache.workspace = torch.empty(need, dtype=torch.uint8, device=dev)
        # the fused step's own workspace: zero-filled once, left zero by every step
        self.step_workspace = torch.zeros(need, dtype=torch.uint8, device=dev) if fused else None
        self.graph = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            # the decode once eagerly on the current contents (no state change)
            self._decode()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        with torch.cuda.graph(self.graph):
            self._step()
        self.graph_fused = None
        if fused:
            self.graph_fused = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.graph_fused):
                self._fused_step()

    def _decode(self) -> None:
        c = self.cache
        kvq.paged_decode_attention(c.cfg, self.q, self.out, c.seq_lens, c.block_tables, c.k_pool, c.v_pool,
                                   c.k_tail, c.v_tail, c.workspace, num_splits=self.num_splits,
                                   num_blocks=c.num_blocks, dev_status=c.dev_status)

    def _step(self) -> None:
        c = self.cache
        kvq.append_tokens(c.cfg, self.new_k, self.new_v, self._cu, c.seq_lens, 1, c.block_tables, c.k_pool,
                          c.v_pool, c.k_tail, c.v_tail, num_blocks=c.num_blocks, dev_status=c.dev_status)
        c.seq_lens.add_(1)
        self._decode()

    def _fused_step(self) -> None:
        c = self.cache
        kvq.append_decode_step(c.cfg, self.new_k, self.new_v, self.q, self.out, c.seq_lens, c.block_tables,
                               c.k_pool, c.v_pool, c.k_tail, c.v_tail, self.step_workspace, self.num_splits,
                               num_blocks=c.num_blocks, dev_status=c.dev_status)

    def completes_tile(self) -> bool:
        """Whether the next step completes a tile of some sequence."""
        c = self.cache
        return bool(np.any((c.host_lens + 1) % c.cfg.tile_tokens == 0))

    def replay(self) -> torch.Tensor:
        c = self.cache
        if np.any(c.host_lens + 1 > c.blocks_per_seq * c.cfg.page_tokens):
            raise ValueError("append past the allocated pages")
        if self.fused and not self.completes_tile():
            self.graph_fused.replay()
        else:
            self.graph.replay()
        c.host_lens = c.host_lens + 1
        return self.out
