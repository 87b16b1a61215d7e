"""Parity at the benchmark's full sizes, in the launch configuration bench.py
times (all heads in one call), on sampled outputs the oracle computes one by
one: the Wan-style 480p workload (all INT4), the HunyuanVideo-style workload
(all INT4) and the 720p workload with every 10th head on the FP16 fallback."""
import numpy as np
import pytest

import oracle
from video_dit_b200 import synth

from gpu_util import accuracy, desc_of, lib, report, row_stats, sm_scale, to_dev

pytestmark = pytest.mark.gpu
TOL = 2e-3


def _head(x, h):
    return np.ascontiguousarray(x[:, h:h + 1])


def _run_full(w, q, k, v, flags):
    import torch
    ra = lib()
    att = ra.RotaAttention(desc_of(w), need_fp16=bool(flags.any()))
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device="cuda")
    att.forward(qd, kd, vd, flags, out)
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    return ra, att, out


def _int4_full_size(name, code_heads, h, tiles):
    """Codes of the sampled heads byte-exact; S and P codes of the sampled row
    tiles of head h bit-exact (same kernel, dump pointers set); outputs of
    those rows within the parity bar of the oracle, with their accuracy."""
    import torch
    w = synth.WORKLOADS[name]
    q, k, v = synth.make_inputs(w)
    flags = w.flags()
    ra, att, out = _run_full(w, q, k, v, flags)
    codes = att.codes()
    for hh in code_heads:                             # prologue codes of sampled heads, byte-exact
        ref = oracle.prepare(_head(q, hh), _head(k, hh), _head(v, hh), w.grid, w.rope_dim, w.had_block, w.theta)
        for key in ("q_codes", "k_codes", "v_codes", "q_scale", "k_scale", "v_scale"):
            got = codes[key][:, hh:hh + 1].cpu().numpy()
            assert np.array_equal(got.view(np.uint8), ref[key].view(np.uint8)), (hh, key)
    ref = oracle.prepare(_head(q, h), _head(k, h), _head(v, h), w.grid, w.rope_dim, w.had_block, w.theta)
    for r0, nr in tiles:
        s = torch.zeros((nr, w.N), dtype=torch.int32, device="cuda")
        p = torch.zeros((nr, w.N), dtype=torch.uint8, device="cuda")
        scratch = torch.empty_like(out)
        ra._check(ra.rota_attn_debug_dump_int4(att.desc, att.buffers, 0, h, r0, nr, s, p, scratch), "dump")
        assert ra.rota_attn_get_error() == ra.ROTA_OK
        o_ref, s_ref, p_ref = oracle.attn_int4(ref, w.N, sm_scale(w), 0, 0, r0, nr, dump=True, group=w.max_group, rowsum=w.row_sum)
        assert np.array_equal(s.cpu().numpy(), s_ref)
        assert np.array_equal(p.cpu().numpy(), p_ref)
        got = out[0, h, r0:r0 + nr].cpu().numpy()
        e, rel, cos = row_stats(got, o_ref)
        report(f"full/{name} h{h} rows {r0}+{nr}",
               accuracy(w, _head(q, h), _head(k, h), _head(v, h), got, o_ref, 0, 0, r0, nr))
        assert e <= TOL, (r0, e, rel, cos)


def test_wan480_full_size_sampled_rows():
    w = synth.WORKLOADS["wan480"]
    _int4_full_size("wan480", (0, 23, w.H - 1), 17, ((w.N // 2 - 64, 128), (w.N - 56, 56)))


def test_hunyuan_full_size_sampled_rows():
    w = synth.WORKLOADS["hunyuan"]
    _int4_full_size("hunyuan", (0, w.H - 1), 9, ((w.N // 3, 128), (w.N - 56, 56)))


def test_wan720_mixed_precision_sampled_rows():
    w = synth.WORKLOADS["wan720"]
    q, k, v = synth.make_inputs(w)
    flags = w.flags()
    assert flags[10] == 1 and flags[11] == 0
    ra, att, out = _run_full(w, q, k, v, flags)
    codes = att.codes()
    # FP16 head 10: RoPE'd rows byte-exact, output rows against textbook attention
    h = 10
    ref = oracle.prepare(_head(q, h), _head(k, h), _head(v, h), w.grid, w.rope_dim, w.had_block, w.theta,
                         np.ones(1, np.uint8))
    got_qr = codes["q_rope"][:, h:h + 1].cpu().numpy().view(np.uint16)
    assert np.array_equal(got_qr, ref["q_rope"])
    for r0, nr in ((0, 32), (w.N - 16, 16)):
        o16 = oracle.attn_fp16(ref["q_rope"], ref["k_rope"], _head(v, h), sm_scale(w), 0, 0, r0, nr)
        e, rel, cos = row_stats(out[0, h, r0:r0 + nr].cpu().numpy(), o16)
        assert e <= TOL, (r0, e, rel, cos)
    # INT4 head 11 of the same call
    h = 11
    ref = oracle.prepare(_head(q, h), _head(k, h), _head(v, h), w.grid, w.rope_dim, w.had_block, w.theta)
    for r0, nr in ((w.N // 3, 32), (w.N - 16, 16)):
        o4 = oracle.attn_int4(ref, w.N, sm_scale(w), 0, 0, r0, nr, group=w.max_group, rowsum=w.row_sum)
        e, rel, cos = row_stats(out[0, h, r0:r0 + nr].cpu().numpy(), o4)
        assert e <= TOL, (r0, e, rel, cos)
