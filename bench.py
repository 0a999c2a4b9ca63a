#!/usr/bin/env python
"""Benchmark of the quantized paged KV-cache hot path on B200.

One step = one pass of the whole path over one batch of the Qwen3-4B-shaped
workload (6 sequences x 131072 cached tokens, 8 KV heads, 32 query heads,
d=128, T=64, 4-bit K and V, n=4):
  1. kvq_quantize_tiles   every full tile of the batch (rotation,
                          normalization, RTN, packing into scattered pages)
  2. kvq_append_tokens    the step's new token per sequence (fp16 tail)
  3. kvq_paged_decode_attention  one decode query per sequence over the
                          packed pages plus the tail (split-K + merge)
With ``--prefill-chunk N`` the line also carries a ``prefill`` object: one
kvq_paged_prefill_attention call per sequence batch, N new tokens per
sequence attending to the whole cache built by the step (quantized tiles
plus tail) and causally to themselves, timed with CUDA events, with its
tensor-core roofline (algorithmic FLOPs: 4 d per query row and visible key).

``value`` is the step's algorithmic bytes (what the method must move: fp16
rows read and packed pages written by 1, tail rows by 2, packed pages,
tables, tail, q and out by 3) per second over the timed steps; the
``decode`` and ``quantize`` objects break it down per call (CUDA events on
the launching stream).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

Under torchrun each rank runs an independent replica batch (weak scaling,
no data-path collective); rank 0 prints one JSON line.  ``--impl
reference`` times the CPU oracle on a bounded sample of the same workload
(rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import math
import multiprocessing as mp
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
METRIC = "paged decode attn GB/s & tok/s over quantized KV (% HBM peak); quantize GB/s"
DECODE_LAUNCHES = 2  # kvq_paged_decode_attention: schedule, tiles (the merge runs inside the tiles kernel)
E2E_CHUNKS = 8  # pieces of the fp16 rows in the end-to-end step (copy of piece k+1 overlaps quantize of piece k)
FALLBACK_HBM_GBS = 6650.0


# --------------------------------------------------------------------------- helpers

def tensor_peak():
    """Dense fp16/bf16 tensor-core TFLOP/s (fp16 runs at the bf16 rate)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return 1590.0, "fallback"


def prefill_flops(ctx_lens, chunk, num_q_heads, d=128):
    """Algorithmic FLOPs of one chunked-prefill call: QK and PV, 2 d each,
    per (query row, visible key); chunk token i of a sequence sees its
    context plus chunk tokens 0..i."""
    keys = 0.0
    for L in ctx_lens:
        keys += chunk * float(L) + chunk * (chunk + 1) / 2.0
    return 4.0 * d * num_q_heads * keys


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# sources a kernel's code depends on (a change to any of them voids its ncu traffic figure)
KERNEL_SOURCES = {
    "quantize_tc_kernel": ("kvq_quantize_tc.cu", "kvq_device.cuh", "kvq_internal.h"),
    "decode_tiles_kernel": ("kvq_decode.cu", "kvq_device.cuh", "kvq_internal.h"),
}


def source_digest(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_paged_kv_tile_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str, units_now: float):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, scaled
    to this launch's units, or None when the kernel changed since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[kernel]
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("source_digest") != source_digest(kernel):
        return None
    return rec["dram_bytes_per_launch"] * units_now / rec["units_per_launch"]


TRAFFIC_UNITS = {
    "quantize_tc_kernel": ("quant_units", "element of the fp16 K/V rows quantized (token x KV head x K|V x channel)"),
    "decode_tiles_kernel": ("decode", "algorithmic byte of the decode call (the byte model's decode figure)"),
}


def record_traffic(csv_path: str, workload: str, num_seqs: int, command: str, out_path: str = None):
    """Write the traffic record of every kernel of KERNEL_SOURCES found in an
    `ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum
    --csv` capture of `command` (run on `workload` with `num_seqs` sequences):
    DRAM bytes per launch (the mean over the captured launches), the units that
    launch processed by the byte model, and the digest of the kernel's sources."""
    import csv
    from quantized_paged_kv_tile_b200 import synth
    with open(csv_path) as f:
        lines = [ln for ln in f if ln.startswith('"')]
    rows = list(csv.DictReader(lines))
    over = {"num_seqs": num_seqs} if num_seqs > 0 else {}
    bm = byte_model(synth.workload(workload, **over), 0, 0)
    out_path = out_path or os.path.join(ROOT, "profiles", "traffic.json")
    rec = {}
    for kernel, (unit_key, unit_text) in TRAFFIC_UNITS.items():
        launches = {}
        for r in rows:
            if kernel in r["Kernel Name"]:
                launches.setdefault(r["ID"], {})[r["Metric Name"]] = float(r["Metric Value"].replace(",", ""))
        if not launches:
            continue
        need = ("dram__bytes_read.sum", "dram__bytes_write.sum", "gpu__time_duration.sum")
        if any(m not in l for l in launches.values() for m in need):
            raise ValueError(f"{csv_path}: a {kernel} launch lacks one of {need}")
        n = len(launches)
        rd = sum(l["dram__bytes_read.sum"] for l in launches.values()) / n
        wr = sum(l["dram__bytes_write.sum"] for l in launches.values()) / n
        rec[kernel] = {"source_digest": source_digest(kernel), "dram_bytes_per_launch": rd + wr,
                       "units_per_launch": bm[unit_key], "unit": unit_text, "capture": command,
                       "launches_captured": n, "dram_bytes_read": rd, "dram_bytes_write": wr,
                       "duration_ns_under_ncu": sum(l["gpu__time_duration.sum"] for l in launches.values()) / n,
                       "workload": f"{workload}, num_seqs={num_seqs or 'default'}"}
    if not rec:
        raise ValueError(f"{csv_path}: no launch of {sorted(TRAFFIC_UNITS)}")
    with open(out_path, "w") as f:
        json.dump(rec, f, indent=1)
        f.write("\n")
    return rec


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        self.path = os.path.join("/tmp", f"kvq_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        load = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(load) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def byte_model(w, cfg_layout_k, cfg_layout_v):
    """Algorithmic bytes of one step (see the module docstring)."""
    d, t, p, h = 128, w.tile_tokens, 16, w.num_kv_heads
    lens0 = np.asarray(w.lens, dtype=np.int64)
    per_tok_head = d * (w.bits_k + w.bits_v) / 8 + 8 + 4 * d / t   # codes + meta + C slices, K+V
    full0 = (lens0 // t) * t
    quant = float(full0.sum()) * h * (2 * d * 2 + per_tok_head)
    rest = lens0 - full0 + w.append_tokens
    append = float(rest.sum()) * h * d * 2 * 2 * 2
    lens1 = lens0 + w.append_tokens
    full1 = (lens1 // t) * t
    tau1 = lens1 - full1
    decode = (float(full1.sum()) * h * per_tok_head + float(full1.sum()) // p * 4
              + float(tau1.sum()) * h * d * 2 * 2 + w.num_seqs * w.num_q_heads * d * 2 * 2)
    return {"quantize": quant, "append": append, "decode": decode, "kv_tokens": float(lens1.sum()),
            "quant_units": float(full0.sum()) * h * 2 * d}


# --------------------------------------------------------------------------- oracle sample

def _oracle_pair(task):
    """One (sequence, KV head) of the workload through the oracle: quantize
    its K and V tiles, dequantize, decode its query group.  Returns bytes."""
    wname, overrides, head, seq = task
    from threadpoolctl import threadpool_limits
    sys.path.insert(0, ROOT)
    from oracle import kvq_oracle as o
    from quantized_paged_kv_tile_b200 import synth
    w = synth.workload(wname, **overrides)
    L0 = w.lens[seq]
    L1 = L0 + w.append_tokens
    with threadpool_limits(1):
        rk = synth.kv_rows_one_head(w, "k", L1, head, stream_id=seq)
        rv = synth.kv_rows_one_head(w, "v", L1, head, stream_id=seq)
        tk, tail_k = o.quantize_sequence(rk, w.tile_tokens, w.bits_k, w.iters)
        tv, tail_v = o.quantize_sequence(rv, w.tile_tokens, w.bits_v, w.iters)
        kh, vh = o.sequence_kv_hat(tk, tail_k), o.sequence_kv_hat(tv, tail_v)
        q = np.random.default_rng(seq * 131 + head).standard_normal((w.group_size, 128))
        o.decode_sequence(q, [kh], [vh], w.group_size)
    return 0


def _warm(_):
    sys.path.insert(0, ROOT)
    import oracle.kvq_oracle  # noqa: F401
    import quantized_paged_kv_tile_b200.synth  # noqa: F401
    return 0


class OraclePool:
    """Spawned worker processes (safe after CUDA init) running oracle pairs."""

    def __init__(self, procs):
        self.procs = procs
        self.pool = mp.get_context("spawn").Pool(procs)
        self.pool.map(_warm, range(procs))

    def time(self, wname, overrides, pairs):
        tasks = [(wname, overrides, h, s) for (s, h) in pairs]
        t0 = time.perf_counter()
        self.pool.map(_oracle_pair, tasks, chunksize=1)
        return time.perf_counter() - t0

    def close(self):
        self.pool.close()
        self.pool.join()


def oracle_pairs(w, n):
    return [(i % w.num_seqs, (i // w.num_seqs) % w.num_kv_heads) for i in range(n)]


def cpu_sample_bytes(w, bm, n_pairs):
    return (bm["quantize"] + bm["append"] + bm["decode"]) * n_pairs / (w.num_seqs * w.num_kv_heads)


# --------------------------------------------------------------------------- GPU arm

def workload_config(w, world: int) -> dict:
    """The `config` object of the JSON line (both arms)."""
    lens0 = np.asarray(w.lens, dtype=np.int64)
    lens1 = lens0 + w.append_tokens
    rows_gb = float(lens0.sum()) * w.num_kv_heads * 128 * 2 * 2 / 1e9
    return {"workload": f"{w.name}: {w.num_seqs} seqs x {int(lens0[0])} cached tokens + {w.append_tokens} appended, "
                        f"{w.num_kv_heads} KV heads, {w.num_q_heads} query heads, d=128, T={w.tile_tokens}, P=16, "
                        f"b_K={w.bits_k}, b_V={w.bits_v}, n={w.iters}, pages scattered by a seeded permutation",
            "global_batch": w.num_seqs * world, "seq_len": int(lens1.max()),
            "parallelism": f"replicas x{world} (no data-path collective)",
            "l2": f"inputs larger than L2 (fp16 rows {rows_gb:.1f} GB per replica)"}


class StepSetup:
    """Device buffers of one workload's step: every full tile of the batch
    quantized (kvq_quantize_tiles), the unfinished prefill rows and the new
    tokens appended (kvq_append_tokens), one decode query per sequence
    (kvq_paged_decode_attention)."""

    def __init__(self, w, dev):
        import torch
        from quantized_paged_kv_tile_b200 import kvq, synth
        self.w = w
        self.dev = dev
        cfg = kvq.Config(num_kv_heads=w.num_kv_heads, group_size=w.group_size, tile_tokens=w.tile_tokens,
                         bits_k=w.bits_k, bits_v=w.bits_v, iters=w.iters)
        self.cfg = cfg
        lay = kvq.get_layout(cfg)
        self.lay = lay
        B, H, T = w.num_seqs, w.num_kv_heads, w.tile_tokens
        lens0 = np.asarray(w.lens, dtype=np.int64)
        lens1 = lens0 + w.append_tokens
        self.lens0, self.lens1 = lens0, lens1
        bps = int(math.ceil(lens1.max() / 16))
        bt_np = synth.block_table(w, bps)
        self.nblocks = int(bt_np.max()) + 1
        self.bt = torch.from_numpy(bt_np).to(dev)
        total0 = int(lens0.sum())
        self.rows_k = synth.kv_rows(w, "k", total0, device=dev)
        self.rows_v = synth.kv_rows(w, "v", total0, device=dev)
        starts = np.concatenate([[0], np.cumsum(lens0)[:-1]])
        full0 = (lens0 // T) * T
        desc_np = np.asarray([(starts[s] + i * T, s, i) for s in range(B) for i in range(lens0[s] // T)],
                             dtype=np.int32).reshape(-1, 3)
        self.desc = torch.from_numpy(desc_np).to(dev)
        # the step's appended rows, contiguous per sequence: the unfinished
        # prefill rows, then the new tokens
        rest = [self.rows_k[starts[s] + full0[s]:starts[s] + lens0[s]] for s in range(B)]
        rest_v = [self.rows_v[starts[s] + full0[s]:starts[s] + lens0[s]] for s in range(B)]
        nk = synth.kv_rows(w, "k", B * w.append_tokens, device=dev, stream_id=1)
        nv = synth.kv_rows(w, "v", B * w.append_tokens, device=dev, stream_id=1)
        a = w.append_tokens
        self.new_k = torch.cat([t for s in range(B) for t in (rest[s], nk[s * a:(s + 1) * a])]).contiguous()
        self.new_v = torch.cat([t for s in range(B) for t in (rest_v[s], nv[s * a:(s + 1) * a])]).contiguous()
        counts = lens1 - full0
        self.cu_new = torch.from_numpy(np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)).to(dev)
        self.before = torch.from_numpy(full0.astype(np.int32)).to(dev)
        self.seq_lens = torch.from_numpy(lens1.astype(np.int32)).to(dev)
        self.k_pool = torch.zeros((self.nblocks, H, lay["page_bytes_k"]), dtype=torch.uint8, device=dev)
        self.v_pool = torch.zeros((self.nblocks, H, lay["page_bytes_v"]), dtype=torch.uint8, device=dev)
        self.k_tail = torch.zeros((B, H, T, 128), dtype=torch.float16, device=dev)
        self.v_tail = torch.zeros_like(self.k_tail)
        self.q = synth.queries(w, device=dev)
        self.out = torch.empty_like(self.q)
        self.ws = torch.empty(kvq.decode_workspace_bytes(cfg, B, 0), dtype=torch.uint8, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.max_new = int(counts.max())
        self.bm = byte_model(w, lay["page_bytes_k"], lay["page_bytes_v"])
        # quantize; append (when there are rows to append); decode = schedule + tiles (the merge runs inside)
        self.launches = (1 if len(desc_np) else 0) + (1 if self.max_new > 0 else 0) + DECODE_LAUNCHES

    def quantize(self, stream, desc=None):
        from quantized_paged_kv_tile_b200 import kvq
        kvq.quantize_tiles(self.cfg, self.rows_k, self.rows_v, self.desc if desc is None else desc, self.bt,
                           self.k_pool, self.v_pool, num_blocks=self.nblocks, dev_status=self.status, stream=stream)

    def append(self, stream):
        from quantized_paged_kv_tile_b200 import kvq
        if self.max_new > 0:  # no unfinished prefill rows and no new tokens: nothing to append
            kvq.append_tokens(self.cfg, self.new_k, self.new_v, self.cu_new, self.before, self.max_new, self.bt,
                              self.k_pool, self.v_pool, self.k_tail, self.v_tail, num_blocks=self.nblocks,
                              dev_status=self.status, stream=stream)

    def decode(self, stream):
        from quantized_paged_kv_tile_b200 import kvq
        kvq.paged_decode_attention(self.cfg, self.q, self.out, self.seq_lens, self.bt, self.k_pool, self.v_pool,
                                   self.k_tail, self.v_tail, self.ws, num_blocks=self.nblocks,
                                   dev_status=self.status, stream=stream)

    def step(self, stream, ev=None):
        if ev is not None:
            ev[0].record(stream)
        self.quantize(stream)
        if ev is not None:
            ev[1].record(stream)
        self.append(stream)
        if ev is not None:
            ev[2].record(stream)
        self.decode(stream)
        if ev is not None:
            ev[3].record(stream)

    def check_status(self, where):
        if int(self.status.item()) != 0:
            raise RuntimeError(f"device status {int(self.status.item())} {where}")


def time_steps(S, stream, steps, warmup):
    """Warm-up, then `steps` timed steps with CUDA events around each call;
    returns per-call millisecond lists and the total."""
    import torch
    for _ in range(warmup):
        S.step(stream)
    torch.cuda.synchronize(S.dev)
    S.check_status("after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        S.step(stream, evs[i])
    t1.record(stream)
    torch.cuda.synchronize(S.dev)
    S.check_status("after the timed steps")
    return {"q": [e[0].elapsed_time(e[1]) for e in evs], "a": [e[1].elapsed_time(e[2]) for e in evs],
            "d": [e[2].elapsed_time(e[3]) for e in evs], "total": t0.elapsed_time(t1)}


def call_objects(S, t, peak):
    """The per-call `decode`, `quantize`, `append` objects of a timed step."""
    w, bm = S.w, S.bm
    q_avg, d_avg = statistics.mean(t["q"]), statistics.mean(t["d"])
    d_gbs = bm["decode"] / (d_avg * 1e-3) / 1e9
    dec = {"gbs": d_gbs, "ms": d_avg, "frac": d_gbs / peak, "tok_per_s": w.num_seqs / (d_avg * 1e-3),
           "kv_tok_per_s": bm["kv_tokens"] / (d_avg * 1e-3), "bytes": bm["decode"],
           "fp16_bytes_equiv": bm["kv_tokens"] * w.num_kv_heads * 512}
    qu = None
    if bm["quantize"] > 0:
        q_gbs = bm["quantize"] / (q_avg * 1e-3) / 1e9
        qu = {"gbs": q_gbs, "ms": q_avg, "frac": q_gbs / peak, "bytes": bm["quantize"]}
    return dec, qu, {"ms": statistics.mean(t["a"]), "bytes": bm["append"]}


def oracle_baseline(wname, w, bm, procs, pairs=None, overrides=None):
    """The oracle (fp64, spawned processes, one BLAS thread each) on a
    bounded sample of (sequence, KV head) pairs of the workload, same byte
    model; with one process it is the single-core figure."""
    pairs = pairs if pairs is not None else oracle_pairs(w, procs)
    pool = OraclePool(procs)
    try:
        secs = pool.time(wname, overrides or {}, pairs)
    finally:
        pool.close()
    per_pair = pair_bytes(w, bm)
    nbytes = float(sum(per_pair[s] for s, _ in pairs))
    return {"value": nbytes / secs / 1e9, "unit": "GB/s", "cores": procs, "kind": "oracle",
            "sample": f"{len(pairs)} of {w.num_seqs * w.num_kv_heads} (sequence, KV head) pairs: fp64 quantize "
                      f"of every K and V tile, dequantize, fp64 decode of the query group; {secs:.1f} s wall on "
                      f"{procs} process{'es' if procs > 1 else ''}, same byte model"}


def pair_bytes(w, bm):
    """Algorithmic step bytes of one (sequence, KV head) pair, per sequence."""
    d, t, p = 128, w.tile_tokens, 16
    per_tok_head = d * (w.bits_k + w.bits_v) / 8 + 8 + 4 * d / t
    lens0 = np.asarray(w.lens, dtype=np.int64)
    lens1 = lens0 + w.append_tokens
    full0, full1 = (lens0 // t) * t, (lens1 // t) * t
    quant = full0 * (2 * d * 2 + per_tok_head)
    append = (lens0 - full0 + w.append_tokens) * d * 2 * 2 * 2
    decode = full1 * per_tok_head + full1 / p * 4 / w.num_kv_heads + (lens1 - full1) * d * 2 * 2 + \
        w.group_size * d * 2 * 2
    return quant + append + decode


def small_pairs(w, n):
    """n (sequence, KV head) pairs over the shortest sequences (a bounded
    oracle sample of a workload with long sequences)."""
    order = np.argsort(np.asarray(w.lens))
    return [(int(order[i % len(order)]), (i // len(order) + i) % w.num_kv_heads) for i in range(n)]


def run_kvq(args, ranks):
    import torch
    from quantized_paged_kv_tile_b200 import build, kvq, synth

    build.build()
    kvq.load_library()
    dev = torch.device("cuda", ranks.local_rank)
    torch.cuda.set_device(dev)
    over = {"num_seqs": args.num_seqs} if args.num_seqs > 0 else {}
    w = synth.workload(args.workload, replica=ranks.rank, **over)
    S = StepSetup(w, dev)
    cfg, B, H = S.cfg, w.num_seqs, w.num_kv_heads
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = hbm_peak()

    for _ in range(args.warmup):
        S.step(stream)
    torch.cuda.synchronize(dev)
    S.check_status("after warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    visible = [x for x in os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",") if x.strip()]
    clocks = ClockSampler(visible[ranks.local_rank] if len(visible) > ranks.local_rank else ranks.local_rank)
    clocks.start()
    ranks.barrier()
    torch.cuda.synchronize(dev)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(args.steps):
        S.step(stream, evs[i])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    ranks.barrier()
    clk = clocks.stop()
    elapsed_ms = t_start.elapsed_time(t_end)
    max_ms = ranks.max(elapsed_ms)
    t = {"q": [e[0].elapsed_time(e[1]) for e in evs], "a": [e[1].elapsed_time(e[2]) for e in evs],
         "d": [e[2].elapsed_time(e[3]) for e in evs]}
    S.check_status("after the timed steps")
    bm = S.bm
    step_bytes = bm["quantize"] + bm["append"] + bm["decode"]
    all_bytes = ranks.sum(step_bytes) * args.steps
    value = all_bytes / (max_ms * 1e-3) / 1e9
    dec, qu, app = call_objects(S, t, peak)
    dec["roofline"] = {"bound": "hbm", "kernel": "decode (schedule + tiles)", "achieved": dec["gbs"],
                       "peak": peak, "peak_kind": peak_kind, "unit": "GB/s", "frac": dec["frac"],
                       "traffic": ncu_traffic("decode_tiles_kernel", bm["decode"])}

    # end to end through the public calls with host buffers.  (1) the whole
    # step: H2D of its inputs (fp16 rows, new rows, q) from pinned memory,
    # the three calls, D2H of the output.  (2) the steady decode step of a
    # serving loop: H2D of the new token rows and q, append + decode, D2H of
    # the output.
    e2e = e2e_decode = None
    if not args.no_e2e:
        host = {name: x.cpu().pin_memory() for name, x in
                dict(rows_k=S.rows_k, rows_v=S.rows_v, new_k=S.new_k, new_v=S.new_v, q=S.q).items()}
        out_host = torch.empty(S.out.shape, dtype=S.out.dtype, pin_memory=True)
        d2h = out_host.numel() * out_host.element_size()

        def e2e_run(names, body, n):
            def one():
                for nm in names:
                    getattr(S, nm).copy_(host[nm], non_blocking=True)
                body()
                out_host.copy_(S.out, non_blocking=True)
            one()
            torch.cuda.synchronize(dev)
            ranks.barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(n):
                one()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            ranks.barrier()
            return ranks.max(e0.elapsed_time(e1)), sum(host[nm].numel() * host[nm].element_size() for nm in names)

        # the step's fp16 rows go up in E2E_CHUNKS pieces on a copy stream; each
        # piece's tiles are quantized as soon as it has landed, so the
        # quantization overlaps the transfer of the next piece (every copy and
        # call is still inside the timed region)
        copy_stream = torch.cuda.Stream(device=dev)
        T = w.tile_tokens
        desc_all = S.desc
        n_desc = int(desc_all.shape[0])
        cuts = [n_desc * c // E2E_CHUNKS for c in range(E2E_CHUNKS + 1)]
        pieces = []
        rows_total = int(S.rows_k.shape[0])
        desc_host = desc_all.cpu().numpy()
        for c in range(E2E_CHUNKS):
            lo_d, hi_d = cuts[c], cuts[c + 1]
            if hi_d <= lo_d:
                continue
            lo = 0 if not pieces else pieces[-1][1]
            hi = rows_total if c == E2E_CHUNKS - 1 else int(desc_host[hi_d - 1, 0]) + T
            pieces.append((lo, hi, desc_all[lo_d:hi_d].clone()))  # own allocation: 16-byte aligned
        if pieces and pieces[-1][1] < rows_total:
            lo, _, d = pieces[-1]
            pieces[-1] = (lo, rows_total, d)

        def step_pipelined():
            start = torch.cuda.Event()
            start.record(stream)
            copy_stream.wait_event(start)
            landed = []
            with torch.cuda.stream(copy_stream):
                for lo, hi, _ in pieces:
                    S.rows_k[lo:hi].copy_(host["rows_k"][lo:hi], non_blocking=True)
                    S.rows_v[lo:hi].copy_(host["rows_v"][lo:hi], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(copy_stream)
                    landed.append(ev)
                for nm in ("new_k", "new_v", "q"):
                    getattr(S, nm).copy_(host[nm], non_blocking=True)
                rest = torch.cuda.Event()
                rest.record(copy_stream)
            for (lo, hi, d), ev in zip(pieces, landed):
                stream.wait_event(ev)
                S.quantize(stream, desc=d)
            stream.wait_event(rest)
            S.append(stream)
            S.decode(stream)
            out_host.copy_(S.out, non_blocking=True)

        n = max(1, min(args.steps, 3))
        step_pipelined()
        torch.cuda.synchronize(dev)
        ranks.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            step_pipelined()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ranks.barrier()
        e_ms = ranks.max(e0.elapsed_time(e1))
        # the pieced step computes what the plain step computes
        piped = out_host.clone()
        S.step(stream)
        torch.cuda.synchronize(dev)
        if not torch.equal(piped, S.out.cpu()):
            raise RuntimeError("the pieced end-to-end step differs from the plain step")
        h2d = sum(host[nm].numel() * host[nm].element_size() for nm in ("rows_k", "rows_v", "new_k", "new_v", "q"))
        e2e = {"value": ranks.sum(step_bytes) * n / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n, "ms_per_step": e_ms / n,
               "what": f"full step with its inputs from pinned host memory: the fp16 rows in {len(pieces)} pieces on a "
                       "copy stream, each piece's tiles quantized once it has landed, then append + decode, output "
                       "back to the host"}
        n = max(3, args.steps)
        e_ms, h2d = e2e_run(("new_k", "new_v", "q"), lambda: (S.append(stream), S.decode(stream)), n)
        dbytes = ranks.sum(bm["append"] + bm["decode"])
        e2e_decode = {"value": dbytes * n / (e_ms * 1e-3) / 1e9, "unit": "GB/s",
                      "tok_per_s": ranks.sum(B) * n / (e_ms * 1e-3), "h2d_bytes_per_step": int(h2d),
                      "d2h_bytes_per_step": int(d2h), "steps": n, "ms_per_step": e_ms / n,
                      "what": "steady serving step: new token rows and q from pinned host memory, append + "
                              "decode, output back to the host"}
        S.check_status("after the end-to-end steps")

    solo = ranks.rank == 0 and ranks.world == 1
    cpu = None
    if solo and not args.no_cpu_baseline:
        procs = max(1, min(os.cpu_count() or 1, 8))
        cpu = oracle_baseline(args.workload, w, bm, procs)
        cpu["single_core"] = oracle_baseline(args.workload, w, bm, 1, pairs=oracle_pairs(w, 1))

    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ranks.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, ranks.world),
        "decode": dec, "quantize": qu, "append": app,
        "roofline": {"bound": "hbm", "kernel": "quantize_tc_kernel", "achieved": qu["gbs"], "peak": peak,
                     "peak_kind": peak_kind, "unit": "GB/s", "frac": qu["frac"],
                     "traffic": ncu_traffic("quantize_tc_kernel", bm["quant_units"])},
        "cpu_baseline": cpu, "e2e": e2e, "e2e_decode_step": e2e_decode,
        "gpu_launches": S.launches * args.steps, "clocks": clk,
    }
    if args.prefill_chunk > 0:
        line["prefill"] = prefill_leg(w, cfg, args, dev, stream, S.seq_lens, S.bt, S.nblocks, S.k_pool, S.v_pool,
                                      S.k_tail, S.v_tail, S.status, S.lens1, cpu_ok=solo)
        line["gpu_launches_prefill"] = args.steps * line["prefill"]["launches_per_call"]
    rows_kv = (S.rows_k, S.rows_v)
    if args.serving_steps > 0:
        line["serving"] = serving_loop(w, cfg, *rows_kv, args.serving_steps, dev)
    del S, rows_kv
    torch.cuda.empty_cache()
    if solo and not args.headline_only and args.workload == "qwen3_4b" and args.num_seqs == 0:
        line["workloads"] = other_workloads(args, dev, stream, peak)
    return line


def other_workloads(args, dev, stream, peak):
    """The other four workloads through the same calls (one GPU, after the
    headline): a few timed steps each (3 warm-up + min(steps, 5) timed), each
    with its own oracle baseline."""
    import torch
    from quantized_paged_kv_tile_b200 import synth
    steps = max(1, min(args.steps, 5))
    procs = max(1, min(os.cpu_count() or 1, 8))
    res = {}
    for name in ("tiny", "mixed", "qwen3_32b_burst"):
        w = synth.workload(name)
        S = StepSetup(w, dev)
        t = time_steps(S, stream, steps, 3)
        dec, qu, app = call_objects(S, t, peak)
        obj = {"config": workload_config(w, 1), "steps": steps, "decode": dec, "quantize": qu, "append": app,
               "step_ms": t["total"] / steps}
        if name == "tiny":
            obj["note"] = "latency-bound: the whole workload fits in L2; a correctness case, not a roofline case"
        if not args.no_cpu_baseline:
            pairs = oracle_pairs(w, procs) if name != "mixed" else small_pairs(w, procs)
            obj["cpu_baseline"] = oracle_baseline(name, w, S.bm, procs, pairs=pairs)
            if name == "mixed":
                obj["cpu_baseline"]["sample"] += " (the shortest sequences)"
        if name == "qwen3_32b_burst":
            obj["serving"] = serving_loop(w, S.cfg, S.rows_k, S.rows_v, w.decode_steps, dev, fused=True)
            obj["serving"]["what"] = (f"{w.decode_steps} steps after the 64 x 16384-token prefill, each one "
                                      f"CUDA-graph replay: kvq_append_decode_step (one launch) on steps that "
                                      f"complete no tile, kvq_append_tokens + kvq_paged_decode_attention on the "
                                      f"tile-completion steps (T = 128), reported apart")
            obj["serving_unfused"] = serving_loop(w, S.cfg, S.rows_k, S.rows_v, w.decode_steps, dev, fused=False)
            obj["serving_unfused"]["what"] = "the same loop with every step as append + length update + decode"
        res[name] = obj
        del S
        torch.cuda.empty_cache()
    res["prefill_sweep"] = prefill_sweep(args, dev, stream, peak, procs)
    return res


def prefill_sweep(args, dev, stream, peak, procs):
    """The 27 (T, b, n) points of the prefill sweep: kvq_quantize_tiles over all
    32 x 16384 new tokens of 8 KV heads, GB/s, and the method's reconstruction
    MSE against plain per-token RTN on a seeded sample of K tiles."""
    import torch
    from quantized_paged_kv_tile_b200 import kvq, synth
    w0 = synth.workload("prefill_sweep")
    total = int(sum(w0.lens))
    rows_k = synth.kv_rows(w0, "k", total, device=dev)
    rows_v = synth.kv_rows(w0, "v", total, device=dev)
    starts = np.concatenate([[0], np.cumsum(w0.lens)[:-1]]).astype(np.int64)
    rng = np.random.default_rng(4444)
    points = []
    for T in (32, 64, 128):
        for b in (2, 3, 4):
            for n in (1, 4, 8):
                w = synth.workload("prefill_sweep", tile_tokens=T, bits_k=b, bits_v=b, iters=n)
                cfg = kvq.Config(num_kv_heads=w.num_kv_heads, group_size=w.group_size, tile_tokens=T, bits_k=b,
                                 bits_v=b, iters=n)
                lay = kvq.get_layout(cfg)
                bps = int(math.ceil(max(w.lens) / 16))
                bt = torch.from_numpy(synth.block_table(w, bps)).to(dev)
                nblocks = w.num_seqs * bps
                k_pool = torch.zeros((nblocks, w.num_kv_heads, lay["page_bytes_k"]), dtype=torch.uint8, device=dev)
                v_pool = torch.zeros((nblocks, w.num_kv_heads, lay["page_bytes_v"]), dtype=torch.uint8, device=dev)
                desc = torch.from_numpy(np.asarray([(starts[s] + i * T, s, i) for s in range(w.num_seqs)
                                                    for i in range(w.lens[s] // T)], dtype=np.int32)).to(dev)
                status = torch.zeros(1, dtype=torch.int32, device=dev)

                def call():
                    kvq.quantize_tiles(cfg, rows_k, rows_v, desc, bt, k_pool, v_pool, num_blocks=nblocks,
                                       dev_status=status, stream=stream)
                for _ in range(2):
                    call()
                torch.cuda.synchronize(dev)
                e = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(3)]
                for e0, e1 in e:
                    e0.record(stream)
                    call()
                    e1.record(stream)
                torch.cuda.synchronize(dev)
                if int(status.item()) != 0:
                    raise RuntimeError(f"device status {int(status.item())} in the sweep at T={T} b={b} n={n}")
                ms = statistics.mean(a.elapsed_time(c) for a, c in e)
                nbytes = byte_model(w, 0, 0)["quantize"]
                gbs = nbytes / (ms * 1e-3) / 1e9
                # reconstruction of sampled K tiles: the GPU's pages read back
                # (original domain) against the fp16 rows, and plain per-token
                # RTN (fp16 scale and zero, no rotation or normalization) of the
                # same rows
                picks = [(int(rng.integers(w.num_seqs)), int(rng.integers(w.lens[0] // T))) for _ in range(4)]
                td = torch.tensor(picks, dtype=torch.int32, device=dev)
                orig = torch.empty((len(picks), w.num_kv_heads, T, 128), dtype=torch.float32, device=dev)
                kvq.unpack_tiles(cfg, td, bt, k_pool, False, out_orig=orig, num_blocks=nblocks, dev_status=status)
                x = torch.stack([rows_k[starts[s] + i * T:starts[s] + (i + 1) * T].permute(1, 0, 2)
                                 for s, i in picks]).double()
                mse_m = float(((orig.double() - x) ** 2).mean())
                mse_p = float(((plain_rtn(x, b) - x) ** 2).mean())
                points.append({"T": T, "b": b, "n": n, "ms": ms, "gbs": gbs, "frac": gbs / peak, "bytes": nbytes,
                               "mse_method": mse_m, "mse_plain_rtn": mse_p, "mse_ratio": mse_m / mse_p})
                del k_pool, v_pool
    head = next(p for p in points if (p["T"], p["b"], p["n"]) == (64, 4, 4))
    res = {"points": points, "headline_point": head,
           "what": "32 seqs x 16384 new tokens, 8 KV heads, K and V, outlier channels 1-5% x[5, 50]; 2 warm-up "
                   "+ 3 timed kvq_quantize_tiles calls per point; MSE on 4 seeded K tiles x 8 heads per point"}
    if not args.no_cpu_baseline:
        res["cpu_baseline"] = oracle_baseline("prefill_sweep", w0, byte_model(w0, 0, 0), procs)
    del rows_k, rows_v
    torch.cuda.empty_cache()
    return res


def plain_rtn(x, bits):
    """Plain per-token asymmetric RTN of fp16 rows x[..., d] (no rotation, no
    normalization): codes from the exact scale, reconstruction with fp16
    scale and zero (the comparator of the method-value check)."""
    import torch
    qmax = (1 << bits) - 1
    z = x.amin(dim=-1, keepdim=True)
    s = (x.amax(dim=-1, keepdim=True) - z) / qmax
    code = torch.where(s > 0, torch.clamp(torch.round((x - z) / torch.where(s > 0, s, torch.ones_like(s))), 0, qmax),
                       torch.zeros_like(x))
    return code * s.half().double() + z.half().double()


def prefill_cpu_sample(w, chunk: int, ctx_tokens: int = 16384, tokens: int = 64):
    """The oracle on a bounded sample of the chunked-prefill workload: one
    (sequence, KV head) with a ``ctx_tokens`` context quantized by the oracle
    (not timed), then, timed, the read path as the oracle states it: the
    context dequantized and fp64 attention of the first ``tokens`` chunk
    tokens x g query heads over it and causally over the chunk rows.
    Returns (algorithmic FLOPs, seconds); one BLAS thread."""
    from threadpoolctl import threadpool_limits
    sys.path.insert(0, ROOT)
    from oracle import kvq_oracle as o
    from quantized_paged_kv_tile_b200 import synth
    tokens = min(tokens, chunk)
    with threadpool_limits(1):
        rk = synth.kv_rows_one_head(w, "k", ctx_tokens + tokens, 0, stream_id=0)
        rv = synth.kv_rows_one_head(w, "v", ctx_tokens + tokens, 0, stream_id=0)
        tk, tail_k = o.quantize_sequence(rk[:ctx_tokens], w.tile_tokens, w.bits_k, w.iters)
        tv, tail_v = o.quantize_sequence(rv[:ctx_tokens], w.tile_tokens, w.bits_v, w.iters)
        q = np.random.default_rng(17).standard_normal((tokens, w.group_size, 128))
        t0 = time.perf_counter()
        kh, vh = o.sequence_kv_hat(tk, tail_k), o.sequence_kv_hat(tv, tail_v)
        o.prefill_chunk_sequence(q, [kh], [vh], rk[ctx_tokens:, None], rv[ctx_tokens:, None], w.group_size)
        secs = time.perf_counter() - t0
    return prefill_flops([ctx_tokens], tokens, w.group_size), secs


def prefill_leg(w, cfg, args, dev, stream, seq_lens, bt, nblocks, k_pool, v_pool, k_tail, v_tail, status, lens1,
                cpu_ok=True):
    """Chunked prefill over the step's cache: every sequence gets
    ``--prefill-chunk`` new tokens attending to its cached tokens and
    causally to themselves (one library call, inputs resident in HBM)."""
    import torch
    from quantized_paged_kv_tile_b200 import kvq, synth
    n = args.prefill_chunk
    B = w.num_seqs
    k_new = synth.kv_rows(w, "k", B * n, device=dev, stream_id=7)
    v_new = synth.kv_rows(w, "v", B * n, device=dev, stream_id=7)
    g = torch.Generator(device=dev)
    g.manual_seed(w.seed * 1000 + 9)
    q = torch.randn((B * n, w.num_q_heads, 128), generator=g, device=dev).to(torch.float16)
    out = torch.empty_like(q)
    cu = torch.arange(0, B * n + 1, n, dtype=torch.int32, device=dev)

    splits = kvq.prefill_splits(cfg, B, n, int(lens1.max()), torch.cuda.get_device_properties(dev).multi_processor_count)
    need = kvq.prefill_workspace_bytes(cfg, B, n, splits)
    ws = torch.empty(need, dtype=torch.uint8, device=dev) if need > 0 else None

    def call():
        kvq.paged_prefill_attention(cfg, q, out, k_new, v_new, cu, seq_lens, n, bt, k_pool, v_pool, k_tail, v_tail,
                                    num_splits=splits, workspace=ws, num_blocks=nblocks, dev_status=status,
                                    stream=stream)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for e0, e1 in evs:
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after the prefill calls")
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    flops = prefill_flops(lens1, n, w.num_q_heads)
    peak, kind = tensor_peak()
    tflops = flops / (ms * 1e-3) / 1e12
    cpu = None
    if not args.no_cpu_baseline and cpu_ok:
        sflops, secs = prefill_cpu_sample(w, n)
        cpu = {"value": sflops / secs / 1e12, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
               "sample": f"1 (sequence, KV head), a 16384-token context quantized by the oracle (untimed), then "
                         f"dequantized and fp64 causal prefill attention of {min(64, n)} chunk tokens x "
                         f"{w.group_size} query heads: {secs:.2f} s on one thread"}
    return {"chunk_tokens": n, "ms": ms, "chunk_tok_per_s": B * n / (ms * 1e-3), "flops": flops,
            "context_splits": splits, "launches_per_call": 1 if splits == 1 else 2, "cpu_baseline": cpu,
            "context": f"{B} seqs x {int(lens1[0])} cached tokens (quantized tiles + fp16 tail)",
            "roofline": {"bound": "tensor", "kernel": "prefill_attn_kernel", "achieved": tflops, "peak": peak,
                         "peak_kind": kind, "unit": "TFLOP/s", "frac": tflops / peak, "traffic": None,
                         "note": "algorithmic FLOPs; the kernel runs each product on hi and lo fp16 halves, "
                                 "so its tensor-core work is twice this"}}


def serving_loop(w, cfg, rows_k, rows_v, steps, dev, fused=False):
    """The serving loop of the workload after its prefill: ``steps`` graph-
    replayed steps of one appended token per sequence plus a decode, each
    timed with CUDA events; tile-completion steps reported apart.  With
    ``fused`` the steps that complete no tile are one launch
    (kvq_append_decode_step)."""
    import torch
    from quantized_paged_kv_tile_b200 import kvq, synth
    from quantized_paged_kv_tile_b200.paged import DecodeStepGraph, PagedKVCache
    lens0 = np.asarray(w.lens, dtype=np.int64)
    bps = int(math.ceil((lens0.max() + steps) / 16))
    cache = PagedKVCache(cfg, w.num_seqs, bps * 16, device=dev, block_table=synth.block_table(w, bps))
    cache.prefill(rows_k, rows_v, lens0)
    splits = kvq.step_splits(cfg, w.num_seqs, torch.cuda.get_device_properties(dev).multi_processor_count)
    graph = DecodeStepGraph(cache, num_splits=splits, fused=fused)
    ms, done = [], []
    for i in range(steps):
        graph.new_k.copy_(synth.kv_rows(w, "k", w.num_seqs, device=dev, stream_id=1 + i))
        graph.new_v.copy_(synth.kv_rows(w, "v", w.num_seqs, device=dev, stream_id=1 + i))
        graph.q.copy_(synth.queries(w, device=dev, step=i))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        graph.replay()
        e1.record()
        ms.append((e0, e1))
        done.append(bool(np.any((lens0 + i + 1) % w.tile_tokens == 0)))
    torch.cuda.synchronize(dev)
    if cache.status() != 0:
        raise RuntimeError(f"device status {cache.status()} in the serving loop")
    t = np.array([a.elapsed_time(b) for a, b in ms])
    comp = t[np.array(done)]
    plain = t[~np.array(done)]
    return {"steps": steps, "graph": True, "fused": fused, "num_splits": splits,
            "launches_per_step": "1 (2 + 1 length update on tile-completion steps)" if fused else
            f"{1 + 1 + DECODE_LAUNCHES} (append, length update, decode)",
            "mean_ms": float(t.mean()), "p50_ms": float(np.percentile(t, 50)),
            "p99_ms": float(np.percentile(t, 99)), "completion_steps": int(comp.size),
            "completion_step_ms": float(comp.mean()) if comp.size else None,
            "other_step_ms": float(plain.mean()) if plain.size else None,
            "decode_tok_per_s": w.num_seqs / (float(t.mean()) * 1e-3)}


# --------------------------------------------------------------------------- reference arm

def run_reference(args, ranks):
    from quantized_paged_kv_tile_b200 import synth
    over = {"num_seqs": args.num_seqs} if args.num_seqs > 0 else {}
    w = synth.workload(args.workload, **over)
    bm = byte_model(w, 0, 0)
    procs = max(1, min(os.cpu_count() or 1, 8))
    pairs = oracle_pairs(w, procs)
    times = []
    pool = OraclePool(procs)
    try:
        for i in range(args.warmup + args.steps):
            secs = pool.time(args.workload, {}, pairs)
            if i >= args.warmup:
                times.append(secs)
    finally:
        pool.close()
    nbytes = cpu_sample_bytes(w, bm, len(pairs))
    value = nbytes * len(times) / sum(times) / 1e9
    sample = (f"per step {len(pairs)} of {w.num_seqs * w.num_kv_heads} (sequence, KV head) pairs: fp64 quantize "
              f"of every K and V tile, dequantize, fp64 decode of the query group, {procs} processes")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ranks.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, ranks.world),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": procs, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kvq", "reference"], default="kvq")
    ap.add_argument("--workload", default="qwen3_4b")
    ap.add_argument("--num-seqs", type=int, default=0,
                    help="override the workload's sequence count (smaller inputs for profiler captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--prefill-chunk", type=int, default=512,
                    help="also time chunked-prefill attention of this many new tokens per sequence over the cache "
                         "(0: off)")
    ap.add_argument("--headline-only", action="store_true",
                    help="only the headline workload (no sub-objects for the other workloads)")
    ap.add_argument("--serving-steps", type=int, default=0,
                    help="after the measurement, time this many graph-replayed append+decode serving steps")
    ap.add_argument("--record-traffic", metavar="CSV",
                    help="write profiles/traffic.json from an ncu --csv capture (dram bytes read/write and duration) "
                         "of the command given by --traffic-command on --workload/--num-seqs, then exit (no GPU)")
    ap.add_argument("--traffic-command", default="")
    args = ap.parse_args()
    if args.record_traffic:
        sys.path.insert(0, ROOT)
        rec = record_traffic(args.record_traffic, args.workload, args.num_seqs, args.traffic_command)
        print(json.dumps({k: v["dram_bytes_per_launch"] for k, v in rec.items()}))
        return 0
    if args.warmup < 3:
        print("warning: fewer than 3 warm-up steps", file=sys.stderr)
    sys.path.insert(0, ROOT)
    from quantized_paged_kv_tile_b200.dist import Ranks

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        if rank != 0:
            return 0
        class _Solo:
            world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
        line = run_reference(args, _Solo())
        print(json.dumps(line), flush=True)
        return 0
    ranks = Ranks()
    if ranks.world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={ranks.world}", file=sys.stderr)
    try:
        line = run_kvq(args, ranks)
        if ranks.rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        ranks.close()
    return 0


if __name__ == "__main__":
    sys.exit(main())
