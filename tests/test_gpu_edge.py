"""GPU parity on the degenerate and extreme inputs of the path: a single
token, the maximum head count, all-zero inputs, an all-zero K block (scale 0,
so c = 0 for that block), V near the fp16 maximum with logits up to the
method's 2^20 range, and very small V (tiny V scales).
Codes and scales byte-exact, S and P codes bit-exact, outputs within max-abs
2e-3 of the oracle's double result."""
import numpy as np
import pytest

import oracle
from video_dit_b200 import synth

from gpu_util import row_stats, run, sm_scale

pytestmark = pytest.mark.gpu

TOL = 2e-3

ONE = synth.Workload("one_token", B=1, H=2, d=64, rope_dim=(16, 24, 24), grid=(1, 1, 1))
MAXH = synth.Workload("max_heads", B=1, H=256, d=64, rope_dim=(16, 24, 24), grid=(1, 2, 9))      # N=18
# the same two shapes in the Wan layout (d = 128, Hadamard 4/2/2): the persistent prologue kernel
ONE_WAN = synth.Workload("one_token_wan", B=1, H=2, d=128, rope_dim=(44, 42, 42), grid=(1, 1, 1))
MAXH_WAN = synth.Workload("max_heads_wan", B=1, H=256, d=128, rope_dim=(44, 42, 42), grid=(1, 2, 9))
SMALL = synth.scaled(synth.WORKLOADS["wan480"], "edge", H=2, grid=(2, 7, 11))                     # N=154


def _scaled_to(x: np.ndarray, peak: float) -> np.ndarray:
    x32 = x.astype(np.float32)
    return (x32 * np.float32(peak / np.abs(x32).max())).astype(np.float16)


def _inputs(case):
    if case == "one_token":
        return ONE, synth.make_inputs(ONE, seed=7)
    if case == "max_heads":
        return MAXH, synth.make_inputs(MAXH, seed=8)
    if case == "one_token_wan":
        return ONE_WAN, synth.make_inputs(ONE_WAN, seed=7)
    if case == "max_heads_wan":
        return MAXH_WAN, synth.make_inputs(MAXH_WAN, seed=8)
    w = SMALL
    q, k, v = synth.make_inputs(w, seed=9)
    if case == "zeros":
        return w, (np.zeros_like(q), np.zeros_like(k), np.zeros_like(v))
    if case == "zero_k_block":
        k = k.copy()
        k[:, :, 64:128] = 0
        return w, (q, k, v)
    if case == "huge":
        # V near the fp16 maximum; Q and K as large as keeps the logits |S c|
        # below 2^20, the range in which the key that sets the running max
        # keeps code 15 (beyond it the fp32 rounding of that max alone can
        # move the key's exponent past log2(14.5 / 15))
        return w, (_scaled_to(q, 1500.0), _scaled_to(k, 1500.0), _scaled_to(v, 60000.0))
    if case == "tiny_v":
        return w, (q, k, _scaled_to(v, 2e-3))
    raise KeyError(case)


CASES = ["one_token", "max_heads", "one_token_wan", "max_heads_wan", "zeros", "zero_k_block", "huge", "tiny_v"]


@pytest.mark.parametrize("case", CASES)
def test_edge_case_parity(case):
    w, (q, k, v) = _inputs(case)
    h = w.H - 1
    codes, out, (s, p, out2) = run(w, q, k, v, dump=(0, h, 0, w.N))
    ref = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block, w.theta, None)
    for key in ("q_codes", "k_codes", "v_codes"):
        assert np.array_equal(codes[key], ref[key]), key
    for key in ("q_scale", "k_scale", "v_scale"):
        assert np.array_equal(codes[key].view(np.uint32), ref[key].view(np.uint32)), key
    o_ref, s_ref, p_ref = oracle.attn_int4(ref, w.N, sm_scale(w), 0, h, 0, w.N, dump=True, group=w.max_group, rowsum=w.row_sum)
    if case == "huge":
        kappa = np.float64(np.float32(np.float64(np.float32(sm_scale(w))) * 1.4426950408889634))
        cmax = np.float64(ref["q_scale"].max()) * np.float64(ref["k_scale"].max()) * kappa
        assert 2.0 ** 16 < np.abs(s_ref).max() * cmax < 2.0 ** 20
    assert np.array_equal(s, s_ref)
    assert np.array_equal(p, p_ref)
    heads = range(w.H) if w.H <= 8 else (0, 1, w.H // 2, w.H - 1)
    for hh in heads:
        o = o_ref if hh == h else oracle.attn_int4(ref, w.N, sm_scale(w), 0, hh, 0, w.N, group=w.max_group, rowsum=w.row_sum)
        assert np.isfinite(out[0, hh]).all(), hh
        e, rel, cos = row_stats(out[0, hh], o)
        assert e <= TOL, (hh, e, rel, cos)
    if case == "zeros":
        assert not out.any()                       # every code 0: O = 0 exactly
    if case in ("one_token", "one_token_wan"):
        # one key: its P code is 15, so O = RN(RN(15 s v) / 15): two fp32
        # roundings away from the key's dequantised V row s v
        sv = ref["v_scale"][0, h, 0].astype(np.float64)
        vc = oracle.unpack_codes(ref["v_codes"][0, h, 0])[:, 0].astype(np.float64)
        assert np.all(np.abs(out[0, h, 0] - sv * vc) <= 2.0 ** -22 * np.abs(sv * vc))
