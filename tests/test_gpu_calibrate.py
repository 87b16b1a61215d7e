"""Choosing the FP16-fallback heads on the GPU: the per-head error kernel
against numpy on the same outputs, and the calibration flagging the heads
whose INT4 output is damaged by planted token outliers (Q/K rows x40 make
their blocks' scales 40 times coarser), with the per-head errors close to the
oracle's INT4-vs-FP16 errors."""
import numpy as np
import pytest

import oracle
from video_dit_b200 import synth

from gpu_util import desc_of, lib, sm_scale, to_dev

pytestmark = pytest.mark.gpu

# plain Gaussians: there INT4 tracks FP16 (relative error ~0.3), so a damaged head stands out
W = synth.scaled(synth.WORKLOADS["wan480"], "calib", H=6, grid=(2, 7, 11), qk_outliers=(0, 0, 0),
                 v_token_frac=0.0)                                                         # N=154
DAMAGED = (1, 4)


def _inputs():
    q, k, v = synth.make_inputs(W, seed=6)
    q, k = q.copy(), k.copy()
    toks = [3, 70, 140]
    for h in DAMAGED:
        q[0, h, toks, :] = (q[0, h, toks, :].astype(np.float32) * 40).astype(np.float16)
        k[0, h, toks, :] = (k[0, h, toks, :].astype(np.float32) * 40).astype(np.float16)
    return q, k, v


def test_head_error_matches_numpy():
    import torch
    ra = lib()
    rng = np.random.default_rng(5)
    shape = (W.B, W.H, W.N, W.d)
    ref = rng.standard_normal(shape).astype(np.float32)
    noise = np.linspace(0.01, 0.3, W.H, dtype=np.float32)[None, :, None, None]
    test = (ref + rng.standard_normal(shape).astype(np.float32) * noise).astype(np.float32)
    sums = torch.full((W.B * W.H * 2,), float("nan"), dtype=torch.float64, device="cuda")
    assert ra.rota_attn_head_error(desc_of(W), to_dev(test), to_dev(ref), sums) == ra.ROTA_OK
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    got = sums.cpu().numpy().reshape(W.B * W.H, 2)
    t64, r64 = test.astype(np.float64).reshape(W.B * W.H, -1), ref.astype(np.float64).reshape(W.B * W.H, -1)
    want = np.stack([((t64 - r64) ** 2).sum(1), (r64 ** 2).sum(1)], 1)
    assert np.allclose(got, want, rtol=1e-12, atol=0)


def test_calibration_flags_the_damaged_heads():
    ra = lib()
    q, k, v = _inputs()
    att = ra.RotaAttention(desc_of(W), need_fp16=True)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    flags, rel = att.calibrate_flags(qd, kd, vd, max_rel_err=0.6)
    assert flags.tolist() == [1 if h in DAMAGED else 0 for h in range(W.H)], rel
    # the same errors from the oracle's INT4 and FP16 paths
    ref4 = oracle.prepare(q, k, v, W.grid, W.rope_dim, W.had_block, W.theta, None)
    ref16 = oracle.prepare(q, k, v, W.grid, W.rope_dim, W.had_block, W.theta, np.ones(W.H, np.uint8))
    for h in range(W.H):
        o4 = oracle.attn_int4(ref4, W.N, sm_scale(W), 0, h, 0, W.N)
        o16 = oracle.attn_fp16(ref16["q_rope"], ref16["k_rope"], v, sm_scale(W), 0, h, 0, W.N)
        want = np.sqrt(((o4 - o16) ** 2).sum() / (o16 ** 2).sum())
        assert abs(rel[h] - want) < 0.02, (h, rel[h], want)
    # a budget of one head keeps one of the two damaged heads
    flags1, _ = att.calibrate_flags(qd, kd, vd, max_rel_err=0.6, max_fp16_heads=1)
    assert flags1.sum() == 1 and int(np.argmax(flags1)) in DAMAGED
    # the chosen flags then drive a normal call
    out = att.forward(qd, kd, vd, flags).cpu().numpy()
    assert ra.rota_attn_get_error() == ra.ROTA_OK and np.isfinite(out).all()
