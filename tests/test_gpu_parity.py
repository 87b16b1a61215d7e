"""GPU parity: the CUDA path against the CPU oracle on the same seeded inputs.

Bars: integer codes, scales, RoPE'd fp16 rows, s32 scores and P codes
bit-exact; attention outputs within max-abs 2e-3 of the oracle's double
result.  Sizes span several 128-row tiles and 64-key blocks with a ragged
tail (N mod 64 != 0), both head dims (64, 128) and all three RoPE splits."""
import math

import numpy as np
import pytest

import oracle
from video_dit_b200 import synth

from gpu_util import accuracy, report, row_stats, run, sm_scale

pytestmark = pytest.mark.gpu

TOL = 2e-3

CASES = {
    "tiny": synth.WORKLOADS["tiny"],                                                  # N=256, d=64
    "wan_mini": synth.scaled(synth.WORKLOADS["wan480"], "wan_mini", H=3, grid=(3, 10, 13)),     # N=390
    "hunyuan_mini": synth.scaled(synth.WORKLOADS["hunyuan"], "hy_mini", H=2, grid=(3, 9, 20)),  # N=540
    "ragged_small": synth.scaled(synth.WORKLOADS["wan480"], "ragged", H=1, grid=(1, 3, 7)),     # N=21 < 64
    # uneven RoPE split: rotation blocks start at channels 42 and 86, off any power-of-two grid
    "offgrid": synth.scaled(synth.WORKLOADS["wan480"], "offgrid", H=2, grid=(2, 7, 11), rope_dim=(42, 44, 42)),
    # rotation blocks of 32 and 64 channels (the largest Hadamard orders)
    "wide_blocks": synth.scaled(synth.WORKLOADS["wan480"], "wide", H=1, grid=(2, 5, 7), rope_dim=(32, 32, 64)),
    # the merged per-pair rotation (a phase in the RoPE tables) in place of the 2-channel
    # Hadamard blocks of the h and w partitions, and on top of the 4-channel ones of t
    "merged_phase": synth.scaled(synth.WORKLOADS["wan480"], "merged", H=2, grid=(3, 10, 13), had=(4, 1, 1),
                                 rope_phase=(0.3, math.pi / 4, -math.pi / 4)),
    # Hadamard blocks of non-power-of-two orders: the whole 44-channel partition (Paley I,
    # q = 43) and the 56-channel ones (Paley II, q = 13, doubled)
    "hadamard_44": synth.scaled(synth.WORKLOADS["wan480"], "h44", H=2, grid=(3, 10, 13), had=(44, 2, 2)),
    "hadamard_56": synth.scaled(synth.WORKLOADS["hunyuan"], "h56", H=2, grid=(3, 9, 20), had=(16, 56, 56)),
    # numerics options: the running max over 128-key groups (two blocks share one max; an odd
    # block count leaves a one-block last group), and the unquantised row sum l = sum 15 * 2^d
    "max_group_128": synth.scaled(synth.WORKLOADS["wan480"], "g128", H=2, grid=(3, 10, 13), max_group=128),
    "max_group_128_even": synth.scaled(synth.WORKLOADS["hunyuan"], "g128e", H=2, grid=(2, 8, 16),
                                       max_group=128),
    "row_sum_r1": synth.scaled(synth.WORKLOADS["wan480"], "r1", H=2, grid=(3, 10, 13), row_sum=1),
    "g128_r1_tiny": synth.scaled(synth.WORKLOADS["tiny"], "g128r1", max_group=128, row_sum=1),
    # head_dim 64 with 8-channel blocks aligned to 16/24/24: the persistent prologue at d = 64
    "tiny_had8": synth.scaled(synth.WORKLOADS["tiny"], "tiny_h8", had=(8, 8, 8)),
}

# Many key blocks per CTA (74), so every pipeline stage and barrier phase wraps many times.
LONG = synth.scaled(synth.WORKLOADS["wan480"], "wan_long", H=2, grid=(3, 30, 52))           # N=4680


def _oracle(w, q, k, v, flags=None):
    return oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block, w.theta, flags, phase=w.rope_phase)


@pytest.mark.parametrize("name", list(CASES))
def test_prologue_codes_bit_exact(name):
    w = CASES[name]
    q, k, v = synth.make_inputs(w)
    codes, _, _ = run(w, q, k, v)
    ref = _oracle(w, q, k, v)
    for key in ("q_codes", "k_codes", "v_codes"):
        assert np.array_equal(codes[key], ref[key]), key
    for key in ("q_scale", "k_scale", "v_scale"):
        assert np.array_equal(codes[key].view(np.uint32), ref[key].view(np.uint32)), key


@pytest.mark.parametrize("name", list(CASES))
def test_int4_scores_and_pcodes_bit_exact(name):
    w = CASES[name]
    q, k, v = synth.make_inputs(w)
    h = w.H - 1
    r0, nr = (0, w.N) if w.N <= 400 else (w.N - 150, 150)
    _, out, (s, p, _) = run(w, q, k, v, dump=(0, h, r0, nr))
    ref = _oracle(w, q, k, v)
    o_ref, s_ref, p_ref = oracle.attn_int4(ref, w.N, sm_scale(w), 0, h, r0, nr, dump=True, group=w.max_group, rowsum=w.row_sum)
    assert np.array_equal(s, s_ref)
    assert np.array_equal(p, p_ref)
    e, rel, cos = row_stats(out[0, h, r0:r0 + nr], o_ref)
    report(f"parity/{name} h{h}", accuracy(w, q, k, v, out[0, h, r0:r0 + nr], o_ref, 0, h, r0, nr))
    assert e <= TOL, (e, rel, cos)


@pytest.mark.parametrize("name", list(CASES))
def test_int4_output_all_heads(name):
    w = CASES[name]
    q, k, v = synth.make_inputs(w)
    _, out, _ = run(w, q, k, v)
    ref = _oracle(w, q, k, v)
    for h in range(w.H):
        o_ref = oracle.attn_int4(ref, w.N, sm_scale(w), 0, h, 0, w.N, group=w.max_group, rowsum=w.row_sum)
        e, rel, cos = row_stats(out[0, h], o_ref)
        assert e <= TOL, (h, e, rel, cos)


@pytest.mark.parametrize("name", ["tiny", "wan_mini", "ragged_small", "merged_phase"])
def test_fp16_fallback_heads(name):
    w = CASES[name]
    q, k, v = synth.make_inputs(w)
    flags = np.zeros(w.H, np.uint8)
    flags[0] = 1
    codes, out, _ = run(w, q, k, v, flags=flags)
    ref = _oracle(w, q, k, v, flags)
    assert np.array_equal(codes["q_rope"][0, 0], ref["q_rope"][0, 0])
    assert np.array_equal(codes["k_rope"][0, 0], ref["k_rope"][0, 0])
    o16 = oracle.attn_fp16(ref["q_rope"], ref["k_rope"], v, sm_scale(w), 0, 0, 0, w.N)
    e, rel, cos = row_stats(out[0, 0], o16)
    assert e <= TOL, (e, rel, cos)
    for h in range(1, w.H):          # the INT4 heads of the same call are unaffected
        o_ref = oracle.attn_int4(ref, w.N, sm_scale(w), 0, h, 0, w.N, group=w.max_group, rowsum=w.row_sum)
        assert row_stats(out[0, h], o_ref)[0] <= TOL


PCODE_ENTRIES = ["rota_attn_debug_pcode", "rota_attn_debug_pcode_fma"]   # exponential on MUFU / on the FMA pipe


@pytest.mark.parametrize("entry", PCODE_ENTRIES)
def test_pcode_function_matches_oracle_dense(entry):
    import torch
    from gpu_util import lib
    ra = lib()
    rng = np.random.default_rng(0)
    d = np.concatenate([rng.uniform(-6, 0, 4_000_000).astype(np.float32),
                        np.float32([-1.0, 0.0, -0.0, -5.0, -4.906890, -30.0, 1e-7])])
    dd = torch.from_numpy(d).cuda()
    u = torch.empty(d.size, dtype=torch.uint8, device="cuda")
    ra._check(getattr(ra, entry)(dd, u), "pcode")
    assert np.array_equal(u.cpu().numpy(), oracle.pcode_array(d))


@pytest.mark.parametrize("entry", PCODE_ENTRIES)
def test_pcode_function_exhaustive_near_thresholds(entry):
    """Every fp32 within 2^16 ulps of each of the 15 code thresholds: the
    band in which the kernel re-decides a code exactly must cover every
    estimate that could round the wrong way."""
    import torch
    from gpu_util import lib
    ra = lib()
    taus = []
    for kk in range(1, 16):
        x = np.float32(np.log2((kk - 0.5) / 15))
        taus.append(x)
    base = np.array(taus, np.float32).view(np.int32)
    offs = np.arange(-(1 << 16), 1 << 16, dtype=np.int32)
    d = (base[:, None] + offs[None, :]).ravel().view(np.float32)
    d = d[d <= 0]
    dd = torch.from_numpy(d).cuda()
    u = torch.empty(d.size, dtype=torch.uint8, device="cuda")
    ra._check(getattr(ra, entry)(dd, u), "pcode")
    assert np.array_equal(u.cpu().numpy(), oracle.pcode_array(d))


def test_int4_long_sequence_sampled_rows():
    w = LONG
    q, k, v = synth.make_inputs(w)
    h, r0, nr = 1, w.N - 200, 200          # the last two CTAs of the head, ragged tail included
    _, out, (s, p, _) = run(w, q, k, v, dump=(0, h, r0, nr))
    ref = _oracle(w, q, k, v)
    o_ref, s_ref, p_ref = oracle.attn_int4(ref, w.N, sm_scale(w), 0, h, r0, nr, dump=True, group=w.max_group, rowsum=w.row_sum)
    assert np.array_equal(s, s_ref)
    assert np.array_equal(p, p_ref)
    e, rel, cos = row_stats(out[0, h, r0:r0 + nr], o_ref)
    report(f"parity/long h{h}", accuracy(w, q, k, v, out[0, h, r0:r0 + nr], o_ref, 0, h, r0, nr))
    assert e <= TOL, (e, rel, cos)
    o0 = oracle.attn_int4(ref, w.N, sm_scale(w), 0, 0, 0, 64, group=w.max_group, rowsum=w.row_sum)          # first rows of the other head
    assert row_stats(out[0, 0, :64], o0)[0] <= TOL


@pytest.mark.parametrize("entry", PCODE_ENTRIES)
def test_pcode_function_exhaustive_range(entry):
    """Every fp32 d in [-6, -0] (about 1.1e9 values): the kernel's P-code
    function against the oracle's, via the oracle's own decision boundaries
    (u(d) is a step function of d, so 15 boundary values pin it everywhere)."""
    import torch
    from gpu_util import lib
    ra = lib()
    lo, hi = 0x80000000, 0xC0C00000            # bit patterns of -0.0 and -6.0; value falls as bits rise

    def val(bits):
        return float(np.uint32(bits).view(np.float32))
    taus = []
    for kk in range(1, 16):                     # most negative d whose oracle code is still >= kk
        a, b = lo, hi                            # code(a) >= kk > code(b)
        while b - a > 1:
            mid = (a + b) // 2
            if oracle.pcode(val(mid)) >= kk:
                a = mid
            else:
                b = mid
        taus.append(val(a))
    tau = torch.tensor(sorted(taus), dtype=torch.float32, device="cuda")
    chunk = 1 << 27
    u = torch.empty(chunk, dtype=torch.uint8, device="cuda")
    for b0 in range(lo, hi + 1, chunk):
        n = min(chunk, hi + 1 - b0)
        bits = torch.arange(b0 - (1 << 32), b0 - (1 << 32) + n, dtype=torch.int32, device="cuda")
        d = bits.view(torch.float32)
        ra._check(getattr(ra, entry)(d, u[:n]), "pcode")
        want = torch.bucketize(d, tau, right=True).to(torch.uint8)
        bad = (u[:n] != want).nonzero()
        assert bad.numel() == 0, (b0, d[bad[:5, 0]].cpu().numpy(), u[bad[:5, 0]].cpu().numpy(),
                                  want[bad[:5, 0]].cpu().numpy())


@pytest.mark.parametrize("base,B,H,grid", [("wan480", 2, 8, (4, 15, 26)), ("tiny", 2, 8, (3, 16, 14))])
def test_prologue_multi_unit_ranges_batch_and_flags(base, B, H, grid):
    """B = 2, H = 8, N = 1560 (25 blocks; d = 128) or N = 672 (11 blocks; d =
    64): 400 / 176 (batch, block, head) units, so CTAs take ranges that cross
    heads, blocks and the batch boundary (at d = 128 more units than the
    persistent CTAs, so ranges of one or two units); heads 3 and 6 are
    flagged (their Q / K come out RoPE'd in fp16, their V job is skipped).
    Codes and scales of the INT4 heads and the RoPE'd rows of the flagged
    heads byte-exact against the oracle."""
    from gpu_util import desc_of, lib, to_dev
    had = (8, 8, 8) if base == "tiny" else None          # d = 64: blocks that fit a chunk
    w = synth.scaled(synth.WORKLOADS[base], "multi_unit_" + base, B=B, H=H, grid=grid,
                     **({"had": had} if had else {}))
    q, k, v = synth.make_inputs(w)
    flags = np.zeros(w.H, np.uint8)
    flags[[3, 6]] = 1
    ra = lib()
    att = ra.RotaAttention(desc_of(w), need_fp16=True)
    att.prepare(to_dev(q), to_dev(k), to_dev(v), flags)
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    codes = {k_: (None if t is None else t.cpu().numpy()) for k_, t in att.codes().items()}
    ref = _oracle(w, q, k, v, flags)
    int4 = [h for h in range(w.H) if not flags[h]]
    for key in ("q_codes", "k_codes", "v_codes"):
        assert np.array_equal(codes[key][:, int4], ref[key][:, int4]), key
    for key in ("q_scale", "k_scale", "v_scale"):
        assert np.array_equal(codes[key][:, int4].view(np.uint32), ref[key][:, int4].view(np.uint32)), key
    for h in (3, 6):
        assert np.array_equal(codes["q_rope"].view(np.uint16)[:, h], ref["q_rope"][:, h]), h
        assert np.array_equal(codes["k_rope"].view(np.uint16)[:, h], ref["k_rope"][:, h]), h
