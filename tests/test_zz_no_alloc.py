"""The allocation-free entry point (rota_attn_fwd_int4_noalloc).

Some callers cannot allocate device memory themselves -- a plugin running
inside an application that owns the device allocator, or a latency-critical
loop where a cudaMalloc could synchronise the device.  For them the library
keeps the intermediate codes in a static device array and takes only the
inputs and the output.  This test calls it through the C ABI twice in a row
(different inputs each time, so stale scratch contents would show) and
checks each result against the regular caller-allocated path
(rota_attn_prepare_qk + rota_attn_fwd_int4): both run the same kernels on
the same codes, so the outputs must be byte-identical.
The file is named so that pytest collects it last."""
import numpy as np
import pytest

from video_dit_b200 import synth

from gpu_util import desc_of, lib, to_dev



@pytest.mark.gpu
def test_noalloc_matches_regular_path_twice():
    """A larger problem first (more heads, longer sequence), then the ragged
    N = 390 one: if the second call read anything the first one left in the
    shared array, its output would differ from the regular path's."""
    import torch
    ra = lib()
    base = synth.WORKLOADS["wan480"]
    big = synth.scaled(base, "noalloc_big", H=4, grid=(3, 15, 20))       # N = 900
    small = synth.scaled(base, "noalloc", H=3, grid=(3, 10, 13))         # N = 390, ragged
    for w, seed in ((big, 3), (small, 0), (small, 7)):
        desc = desc_of(w)
        att = ra.RotaAttention(desc, need_fp16=False)
        q, k, v = synth.make_inputs(w, seed=seed)
        qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
        ref = att.forward(qd, kd, vd)
        got = torch.full_like(ref, float("nan"))
        ra._check(ra.rota_attn_fwd_int4_noalloc(desc, qd, kd, vd, got), "fwd_int4_noalloc")
        assert ra.rota_attn_get_error() == ra.ROTA_OK
        # the same kernels on the same codes: byte-identical outputs
        assert torch.equal(got.view(torch.int32), ref.view(torch.int32)), (w.name, seed)


@pytest.mark.gpu
def test_noalloc_rejects_oversize_problem():
    import torch
    ra = lib()
    w = synth.WORKLOADS["wan480"]                 # needs far more than the static scratch
    desc = desc_of(w)
    x = torch.zeros(16, dtype=torch.float16, device="cuda")
    out = torch.zeros(16, dtype=torch.float32, device="cuda")
    assert ra.rota_attn_fwd_int4_noalloc(desc, x, x, x, out) == ra.ROTA_ERR_UNSUPPORTED
