"""Host-side helpers of bench.py on CPU: the DRAM traffic figure reported in
the roofline record scales with the units one launch processes, and is null
where no capture of that kernel instantiation exists."""
import dataclasses
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from video_dit_b200 import synth  # noqa: E402


def test_traffic_scales_with_batch_heads_and_tokens():
    w = synth.WORKLOADS["wan480"]
    per = bench.TRAFFIC_PER_HEAD_TOKEN["attn_int4_kernel"]
    assert bench.traffic_per_launch("attn_int4_kernel", w, 40) == per * w.B * 40 * w.N
    w2 = dataclasses.replace(w, B=2)
    assert bench.traffic_per_launch("attn_int4_kernel", w2, 40) == 2 * bench.traffic_per_launch(
        "attn_int4_kernel", w, 40)
    assert bench.traffic_per_launch("attn_int4_kernel", w, 20) * 2 == bench.traffic_per_launch(
        "attn_int4_kernel", w, 40)


def test_traffic_null_without_a_capture():
    w = synth.WORKLOADS["wan480"]
    assert bench.traffic_per_launch("attn_int4_kernel", w, 0) is None
    assert bench.traffic_per_launch("no_such_kernel", w, 40) is None
    # the P-code variants run other instantiations of the INT4 kernel
    assert bench.traffic_per_launch("attn_int4_kernel", synth.WORKLOADS["wan480_g128"], 40) is None
    assert bench.traffic_per_launch("attn_int4_kernel", synth.WORKLOADS["wan480_r1"], 40) is None
    # the FP16 fallback's figure does not depend on the INT4 numerics options
    assert bench.traffic_per_launch("attn_fp16_kernel", synth.WORKLOADS["wan480_g128"], 4) is not None
