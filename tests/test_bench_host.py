"""Host-side logic of the benchmark that needs no GPU: the routing sample, the
workload description both arms print, and the reference arm's line."""
import json
import subprocess
import sys
import os

import numpy as np

import bench
from chunk_adaptive_mixed_b200 import workloads as W


def test_route_sample_spreads_over_the_batch():
    for N, count in ((512, 128), (4608, 128), (16, 128), (1, 8), (1024, 8)):
        c = bench.route_sample_chunks(N, count)
        assert c == sorted(set(c))
        assert all(0 <= x < N for x in c)
        assert len(c) <= max(min(count, N), 1)
        assert 0 in c and N - 1 in c
        if N >= 4 * count:
            # groups cover the whole batch: no half of it is left out
            assert min(c) < N // 4 and max(c) >= 3 * N // 4


def test_both_arms_print_the_same_config():
    w = W.get("llama2_13b_128k")
    lens = W.seq_lens(w, 0)
    a = bench.line_config(w, lens, True, "moqae", 0.0, False, False, 1)
    b = bench.line_config(w, lens, True, "moqae", 0.0, False, False, 1)
    assert a == b
    assert a["workload"] == "llama2_13b_128k" and a["layers"] == 40
    assert "only the packed cache" in a["kv"]
    assert "sum of the library spans" in a["step_time"]
    small = bench.line_config(W.get("llama2_7b_layer"), W.seq_lens(W.get("llama2_7b_layer"), 0),
                              True, "moqae", 0.0, False, False, 1)
    assert small["l2"].startswith("2 x L2 buffer")


def test_default_workload_is_the_largest_single_gpu_config():
    assert bench.DEFAULT_WORKLOAD == "llama2_13b_128k"
    assert W.get(bench.DEFAULT_WORKLOAD).kv_streamed


def test_reference_arm_line_on_a_small_workload():
    # the oracle on a bounded sample: ms_per_step is the sample's measured
    # time, the value its projection to the full step, the config the same
    # dict our arm prints
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], cwd=root, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "tokens/s"
    w = W.get("tiny")
    assert line["config"] == json.loads(json.dumps(
        bench.line_config(w, W.seq_lens(w, 0), True, "moqae", 0.0, False, False, 1)))
    assert line["ms_per_step"] <= line["projected_ms_per_full_step"] + 1e-9
    assert line["sample_wall_s"] * 1e3 >= line["ms_per_step"] * line["steps"] * 0.99
    assert np.isfinite(line["value"]) and line["value"] > 0


def test_pack_traffic_only_for_the_captured_kernel_and_workload():
    # roofline.traffic comes from an ncu capture of one pack.cu on one
    # workload; any other source, workload or map setting reports null
    class S:
        router, lam, rs = "moqae", 0.0, True
    for name, cap in bench.PACK_TRAFFIC.items():
        w = W.get(name)
        want = cap["bytes_per_launch"] if bench.pack_sources_sha256() == cap["sha256"] else None
        assert bench.pack_traffic(w, S, 0) == want
        assert bench.pack_traffic(w, S, 1) is None            # another seed, another map
        S.lam = 1.0
        assert bench.pack_traffic(w, S, 0) is None
        S.lam = 0.0
    assert bench.pack_traffic(W.get("tiny"), S, 0) is None


def test_launch_counts_match_the_committed_launch_lists():
    # the ncu launch lists under profiles/ count every library kernel over
    # 1 warm-up + N timed steps plus one extra routing (prepack, router, vote,
    # 2 layout kernels) that sizes the packed buffers
    extra = 5
    w13 = W.get("llama2_13b_128k")
    assert bench.decode_kernels_per_call(w13) == 3     # prep + decode + merge
    assert 3 * bench.launches_per_step(w13, 1, "moqae") + extra == 500
    w7 = W.get("llama2_7b_32l")
    assert 3 * bench.launches_per_step(w7, 1, "moqae") + extra == 404
    wg = W.get("llama3_8b_gqa")
    assert 2 * bench.launches_per_step(wg, 1, "moqae") + extra == 617
    # fp32 queries (the CUDA-core decode): decode + merge
    wt = W.get("tiny")
    assert bench.decode_kernels_per_call(wt) == 2
    assert bench.launches_per_step(wt, 1, "similarity") == 3 + 1 + 2
    # a split context: partial decode call + combine per layer and step
    assert bench.launches_per_step(w13, 1, "moqae", split=True) == 5 + 40 + 4 * 40


def test_setup_counts_through_the_same_function():
    # the method the bench line uses, on a stand-in with Setup's attributes
    import types
    w = W.get("llama3_8b_gqa")
    s = types.SimpleNamespace(w=w, routers=[None], router="moqae", grow=False, fills=[],
                              shard=None)
    assert bench.Setup.launches_per_step(s) == bench.launches_per_step(w, 1, "moqae") == 306
    s.grow, s.fills = True, [0, 3, 0, 1]
    assert bench.Setup.launches_per_step(s) == 5 + 1 + 100 * (2 + 4) + 2 * (3 + 1)
