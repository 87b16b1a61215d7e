"""Bounded waits: an injected missing MMA makes every wait on it run out; the
kernel exits, the host reads ROTA_ERR_TIMEOUT, and the context stays usable."""
import numpy as np
import pytest

from video_dit_b200 import synth

from gpu_util import desc_of, lib, to_dev

pytestmark = pytest.mark.gpu


def test_injected_timeout_is_reported_and_context_survives():
    import torch
    ra = lib()
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.make_inputs(w)
    att = ra.RotaAttention(desc_of(w), need_fp16=False)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out = torch.zeros((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    att.prepare(qd, kd, vd)
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    ra.rota_attn_debug_inject_timeout(True, 50_000_000)      # 50 ms
    ra._check(ra.rota_attn_fwd_int4(att.desc, att.buffers, None, out), "fwd")
    assert ra.rota_attn_get_error() == ra.ROTA_ERR_TIMEOUT
    # the next call is normal and correct
    out2 = att.forward(qd, kd, vd)
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    assert torch.isfinite(out2).all()
