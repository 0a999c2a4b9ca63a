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


def test_plain_rtn_comparator_matches_the_oracle():
    # bench.py computes the sweep's plain-RTN MSE with torch on the device;
    # on the CPU it must equal the oracle's plain_rtn_baseline exactly
    import numpy as np
    import torch
    import bench
    from oracle import kvq_oracle as o
    rng = np.random.default_rng(12)
    for bits in (2, 3, 4):
        x = (rng.standard_normal((64, 128)) * rng.uniform(0.1, 30, size=(64, 1))).astype(np.float16)
        got = bench.plain_rtn(torch.from_numpy(x).double(), bits).numpy()
        np.testing.assert_array_equal(got, o.plain_rtn_baseline(x, bits))


def test_pair_bytes_add_up_to_the_step():
    # per-(sequence, KV head) bytes summed over every pair give the step's bytes
    import numpy as np
    import bench
    from quantized_paged_kv_tile_b200 import synth
    for name in ("qwen3_4b", "mixed", "qwen3_32b_burst", "tiny"):
        w = synth.workload(name)
        bm = bench.byte_model(w, 0, 0)
        total = bm["quantize"] + bm["append"] + bm["decode"]
        per = bench.pair_bytes(w, bm)
        assert abs(float(np.sum(per)) * w.num_kv_heads - total) <= 1e-9 * total, name


def test_record_traffic_reads_an_ncu_csv(tmp_path):
    # two decode launches and one quantize launch in ncu's --csv layout (with a
    # profiler line mixed in): per-launch means, units from the byte model
    import json
    import bench
    from quantized_paged_kv_tile_b200 import synth
    head = '"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",' \
           '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n'
    rows = []
    for i, (kern, rd, wr, ns) in enumerate([("quantize_tc_kernel<64, 4, 4>", 100, 20, 7),
                                             ("decode_tiles_kernel<64, 4, 4>", "1,000", 10, 3),
                                             ("decode_tiles_kernel<64, 4, 4>", "3,000", 30, 5)]):
        for m, v in (("dram__bytes_read.sum", rd), ("dram__bytes_write.sum", wr), ("gpu__time_duration.sum", ns)):
            rows.append(f'"{i}","1","python3","h","void {kern}(Args)","1","7","(128, 1, 1)","(444, 1, 1)","0",'
                        f'"10.0","Command line profiler metrics","{m}","byte","{v}"\n')
    p = tmp_path / "cap.csv"
    p.write_text("==PROF== Connected to process 1\n" + head + "".join(rows))
    out = tmp_path / "traffic.json"
    rec = bench.record_traffic(str(p), "qwen3_4b", 1, "cmd", str(out))
    bm = bench.byte_model(synth.workload("qwen3_4b", num_seqs=1), 0, 0)
    assert rec["quantize_tc_kernel"]["dram_bytes_per_launch"] == 120
    assert rec["decode_tiles_kernel"]["dram_bytes_per_launch"] == 2000 + 20
    assert rec["decode_tiles_kernel"]["launches_captured"] == 2
    assert rec["quantize_tc_kernel"]["units_per_launch"] == bm["quant_units"]
    assert rec["decode_tiles_kernel"]["units_per_launch"] == bm["decode"]
    assert json.loads(out.read_text()) == rec
    # the record scales to another launch by units, and only while the sources are unchanged
    assert rec["decode_tiles_kernel"]["source_digest"] == bench.source_digest("decode_tiles_kernel")
