"""CPU checks of bench.py's algorithmic work models."""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def test_prefill_flops_counts_visible_keys():
    import bench
    ctx, n, hq, d = [5, 0, 17], 4, 3, 128
    # brute force: every (sequence, chunk token, query head) sees ctx + i + 1 keys, 4 d FLOPs each
    want = sum(4 * d * (c + i + 1) for c in ctx for i in range(n) for _ in range(hq))
    assert bench.prefill_flops(ctx, n, hq, d) == want


def test_tensor_peak_reads_measured_file():
    import json
    import bench
    peak, kind = bench.tensor_peak()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        assert kind == "measured" and peak == float(json.load(open(path))["bf16_tflops"])
    else:
        assert kind == "fallback"


def test_prefill_cpu_sample_runs_the_oracle():
    import bench
    from quantized_paged_kv_tile_b200 import synth
    w = synth.workload("qwen3_4b")
    flops, secs = bench.prefill_cpu_sample(w, 512, ctx_tokens=128, tokens=4)
    assert flops == bench.prefill_flops([128], 4, w.group_size) and secs > 0
