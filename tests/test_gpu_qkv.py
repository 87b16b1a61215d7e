"""GPU parity of the fused QKV projection + prologue (rota_attn_qkv_prepare).

The projection's fp32 accumulation order is not fixed by the method, so the
byte-exact cases use inputs on the grids k / 16 and j / 64, for which every
order gives the same fp32 sum: then the fused path's codes, scales, RoPE'd fp16
rows and fp16 V must equal the oracle's (its projection, rounded to fp16, then
its prologue) bit for bit.  On general fp16 inputs the sums can differ in the
last fp32 bits between orders, so only the share of identical codes is
checked there."""
import numpy as np
import pytest

import oracle
from video_dit_b200 import synth

from gpu_util import desc_of, lib, to_dev

pytestmark = pytest.mark.gpu

CASES = {
    # Wan 44/42/42 (Hadamard 4/2/2) with planted outlier rows in W_q / W_k, ragged tail, 4 tiles
    "wan": (synth.scaled(synth.WORKLOADS["wan480"], "qkv_wan", H=2, grid=(3, 10, 13)), 256),
    # head_dim 64, 16/24/24
    "tiny": (synth.WORKLOADS["tiny"], 128),
    # HunyuanVideo 16/56/56 with 56-channel Hadamard blocks (the dense rotation pass), B = 2
    "hunyuan_h56": (synth.scaled(synth.WORKLOADS["hunyuan"], "qkv_hy", B=2, H=1, grid=(2, 5, 13),
                                 had=(16, 56, 56)), 192),
    # H = 59, C = 1024: the heads' W rows (46 MB) exceed one raster group, so the
    # kernel runs two groups, of 30 and 29 heads.  N = 26 (one ragged tile per
    # head) keeps the oracle's projection short; outlier rows x4 keep the
    # exact-grid sums below 2^24 units.
    "wan_groups": (synth.scaled(synth.WORKLOADS["wan480"], "qkv_groups", H=59, grid=(1, 2, 13), qk_scale=4.0),
                   1024),
}


def _run(w, C, x, wt, flags):
    import torch
    ra = lib()
    att = ra.RotaAttention(desc_of(w), need_fp16=bool(flags.any()))
    v_out = torch.zeros((w.B, w.H, w.N, w.d), dtype=torch.float16, device="cuda")
    ra._check(ra.rota_attn_qkv_prepare(att.desc, to_dev(x), to_dev(wt), C, flags, att.buffers, v_out), "qkv")
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    codes = {k: (None if t is None else t.cpu().numpy()) for k, t in att.codes().items()}
    return att, codes, v_out.cpu().numpy()


@pytest.mark.parametrize("name", list(CASES))
def test_fused_projection_codes_bit_exact(name):
    w, C = CASES[name]
    x, wt = synth.make_qkv_inputs(w, C, seed=3, exact=True)
    flags = np.zeros(w.H, np.uint8)
    _, codes, _ = _run(w, C, x, wt, flags)
    q, k, v = oracle.qkv_project(x, wt, w.H, w.d)
    ref = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block, w.theta, flags, phase=w.rope_phase)
    for key in ("q_codes", "k_codes", "v_codes"):
        assert np.array_equal(codes[key], ref[key]), key
    for key in ("q_scale", "k_scale", "v_scale"):
        assert np.array_equal(codes[key].view(np.uint32), ref[key].view(np.uint32)), key


def test_fused_projection_flagged_head_and_attention():
    """Head 0 flagged: its RoPE'd fp16 Q / K rows and its fp16 V come out of the
    fused call byte-exact; head 1's codes too; and the attention run on the fused
    call's buffers equals the attention on the oracle's codes."""
    import torch
    w, C = CASES["wan"]
    x, wt = synth.make_qkv_inputs(w, C, seed=4, exact=True)
    flags = np.array([1, 0], np.uint8)
    att, codes, v_out = _run(w, C, x, wt, flags)
    q, k, v = oracle.qkv_project(x, wt, w.H, w.d)
    ref = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block, w.theta, flags, phase=w.rope_phase)
    assert np.array_equal(codes["q_rope"].view(np.uint16)[0, 0], ref["q_rope"][0, 0])
    assert np.array_equal(codes["k_rope"].view(np.uint16)[0, 0], ref["k_rope"][0, 0])
    assert np.array_equal(v_out[0, 0].view(np.uint16), v[0, 0].view(np.uint16))
    for key in ("q_codes", "k_codes", "v_codes"):
        assert np.array_equal(codes[key][0, 1], ref[key][0, 1]), key
    ra = lib()
    out = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.float32, device="cuda")
    ra._check(ra.rota_attn_fwd_int4(att.desc, att.buffers, flags, out), "int4")
    ra._check(ra.rota_attn_fwd_fp16_fallback(att.desc, att.buffers, torch.from_numpy(v_out).cuda(), flags, out), "f16")
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    sm = float(np.float32(1 / np.sqrt(w.d)))
    o4 = oracle.attn_int4(ref, w.N, sm, 0, 1, 0, w.N)
    assert np.abs(out[0, 1].cpu().numpy() - o4).max() <= 2e-3
    o16 = oracle.attn_fp16(ref["q_rope"], ref["k_rope"], v, sm, 0, 0, 0, w.N)
    assert np.abs(out[0, 0].cpu().numpy() - o16).max() <= 2e-3


def test_fused_projection_general_inputs():
    """General fp16 inputs: the fp32 sums may differ in their last bits from
    the oracle's correctly rounded ones, which can move a rounding to fp16 and
    then a code by one; nearly all codes agree."""
    w, C = CASES["wan"]
    x, wt = synth.make_qkv_inputs(w, C, seed=6, exact=False)
    flags = np.zeros(w.H, np.uint8)
    _, codes, _ = _run(w, C, x, wt, flags)
    q, k, v = oracle.qkv_project(x, wt, w.H, w.d)
    ref = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block, w.theta, flags, phase=w.rope_phase)
    from codes import unpack
    for key in ("q_codes", "k_codes"):
        a, b = unpack(codes[key]).astype(np.int32), unpack(ref[key]).astype(np.int32)
        assert np.mean(a == b) > 0.99, key
        assert np.abs(a - b).max() <= 1, key


def test_fused_projection_rejects_bad_arguments():
    import torch
    ra = lib()
    w, C = CASES["wan"]
    att = ra.RotaAttention(desc_of(w), need_fp16=False)
    x = torch.zeros((w.B, w.N, C), dtype=torch.float16, device="cuda")
    wt = torch.zeros((3 * w.H * w.d, C), dtype=torch.float16, device="cuda")
    assert ra.rota_attn_qkv_prepare(att.desc, x, wt, 100, None, att.buffers) == ra.ROTA_ERR_INVALID_ARG
    assert ra.rota_attn_qkv_prepare(att.desc, x, wt, 0, None, att.buffers) == ra.ROTA_ERR_INVALID_ARG
    flags = np.array([1, 0], np.uint8)          # a flagged head needs q_rope / k_rope / v_out
    assert ra.rota_attn_qkv_prepare(att.desc, x, wt, C, flags, att.buffers) == ra.ROTA_ERR_INVALID_ARG
