"""Crafted codes that drive the INT4 kernel's rare paths, checked bit-exactly.

The codes and scales are written straight into the library's buffers (no
prologue), so the scores can be placed where the range-optimised P code
decision is hardest: keys whose exponent d = RN(S c - m) lies within a tiny
fraction of a code unit of a threshold 15 * 2^d = k + 1/2 (the kernel flags
them and re-decides them against the exact threshold table, patching the codes
it already stored), the exact tie d = -1 (15 * 2^-1 = 7.5 rounds to the even
code 8), a running max that rises in every key block on every row (O is
rescaled every block), and a ragged last block.  S and the P codes must equal
the oracle's bit for bit; the outputs must agree within the parity tolerance.
"""
import math

import numpy as np
import pytest

import oracle
from video_dit_b200 import synth

from gpu_util import desc_of, lib, row_stats
from gpu_util import kappa as gpu_kappa

TOL = 2e-3
pytestmark = pytest.mark.gpu


def _ulp_step(x: np.float32, k: int) -> np.float32:
    return np.array([x], np.float32).view(np.int32).__add__(np.int32(k)).view(np.float32)[0]


def _c_of(sk, kappa):
    """The score scale both sides use with query scale 1: RN(RN(1 * s_k) kappa)."""
    return np.float32(np.float32(np.float32(1.0) * sk) * kappa)


def _d_of(s_int, c, m):
    """RN(S c - m): S c - m is exact in double, so this is the single rounding of the fma."""
    return np.float32(np.float64(s_int) * np.float64(c) - np.float64(m))


def _gap(d):
    """Distance of 15 * 2^d from the nearest half-integer, in code units."""
    x = 15.0 * 2.0 ** float(d)
    return abs(x - (math.floor(x) + 0.5))


def _tune(kappa, smax, k_code, span=3000):
    """A key scale for which a key one below the block max smax (query code 1)
    lands as close as fp32 allows to the threshold between codes k and k+1."""
    c_target = -math.log2((k_code + 0.5) / 15.0)          # d = -c for S = smax - 1
    base = np.float32(c_target / float(kappa))
    best = None
    for step in range(-span, span):
        sk = _ulp_step(base, step)
        c = _c_of(sk, kappa)
        m = np.float32(np.float64(smax) * np.float64(c))
        g = _gap(_d_of(smax - 1, c, m))
        if best is None or g < best[0]:
            best = (g, sk)
    return best[1], best[0]


def test_near_threshold_codes_rescales_and_exact_tie():
    import torch
    ra = lib()
    d, N = 64, 250                              # 4 key blocks, the last one ragged (58 keys)
    nblk = (N + 63) // 64
    npad = nblk * 64
    w = synth.Workload("crafted", B=1, H=1, d=d, rope_dim=(16, 24, 24), grid=(1, 5, 50))
    assert w.N == N
    desc = desc_of(w)
    sm = float(np.float32(1 / math.sqrt(d)))
    kappa = np.float32(gpu_kappa(d))
    rng = np.random.default_rng(11)

    # Q: channel 0 only, 1 on even rows and 2 on odd rows.  K: channel 0 carries
    # the scores; block j holds its max smax[j] and keys 1..4 below it.  With the
    # scales below the block maxima S c rise block by block on every row.
    smax = [2, 2, 4, 3]
    thresholds = {0: 14, 1: 10, 3: 3}           # k: the tuned keys sit between codes k and k + 1
    q = np.zeros((1, 1, npad, d), np.int32)
    q[0, 0, :N, 0] = np.where(np.arange(N) % 2 == 0, 1, 2)
    k = np.zeros((1, 1, npad, d), np.int32)
    for j in range(nblk):
        n = rng.integers(0, 5, 64)
        n[0] = 0
        n[1:9] = 1
        k[0, 0, 64 * j:64 * (j + 1), 0] = smax[j] - n
    k[0, 0, 128 + 9:128 + 20, 0] = smax[2] - 2  # d = -2 * 0.5 = -1 exactly on even rows
    k[0, 0, N:, :] = 0

    sk = np.ones(nblk, np.float32)
    gaps = {}
    for j, kc in thresholds.items():
        sk[j], gaps[j] = _tune(kappa, smax[j], kc)
    assert max(gaps.values()) < 2e-6, gaps      # inside the kernel's near-tie band with margin
    base = np.float32(0.5 / float(kappa))
    sk[2] = next(_ulp_step(base, s) for s in sorted(range(-64, 65), key=abs)
                 if _c_of(_ulp_step(base, s), kappa) == np.float32(0.5))
    xmax = [float(smax[j]) * float(_c_of(sk[j], kappa)) for j in range(nblk)]
    assert all(a < b for a, b in zip(xmax, xmax[1:])), xmax

    q_scale = np.ones((1, 1, nblk), np.float32)
    k_scale = sk.reshape(1, 1, nblk)
    v = rng.integers(-7, 8, (1, 1, nblk, d, 64)).astype(np.int32)
    v[0, 0, nblk - 1, :, N - 64 * (nblk - 1):] = 0
    v_scale = rng.uniform(0.05, 2.0, (1, 1, nblk, d)).astype(np.float32)

    prep = dict(q_codes=oracle.pack_codes(q), k_codes=oracle.pack_codes(k),
                q_scale=q_scale, k_scale=k_scale, v_codes=oracle.pack_codes(v), v_scale=v_scale)
    o_ref, s_ref, p_ref = oracle.attn_int4(prep, N, sm, 0, 0, 0, N, dump=True)
    assert (p_ref[0::2, 128 + 9:128 + 20] == 8).all()   # the exact tie takes the even code

    att = ra.RotaAttention(desc, need_fp16=False)
    views = att.codes()
    for name, arr in prep.items():
        views[name].copy_(torch.from_numpy(np.ascontiguousarray(arr)).reshape(views[name].shape))
    out = torch.full((1, 1, N, d), float("nan"), dtype=torch.float32, device="cuda")
    ra._check(ra.rota_attn_fwd_int4(desc, att.buffers, None, out), "fwd_int4")
    s = torch.zeros((N, N), dtype=torch.int32, device="cuda")
    p = torch.zeros((N, N), dtype=torch.uint8, device="cuda")
    out2 = torch.empty_like(out)
    ra._check(ra.rota_attn_debug_dump_int4(desc, att.buffers, 0, 0, 0, N, s, p, out2), "dump")
    st = ra.rota_attn_get_error()
    assert st == ra.ROTA_OK, ra.rota_attn_status_string(st)

    assert np.array_equal(s.cpu().numpy(), s_ref)
    p_got = p.cpu().numpy()
    bad = np.argwhere(p_got != p_ref)
    assert bad.size == 0, [(int(i), int(c), int(p_got[i, c]), int(p_ref[i, c])) for i, c in bad[:8]]
    for got in (out.cpu().numpy()[0, 0], out2.cpu().numpy()[0, 0]):
        e, rel, cos = row_stats(got, o_ref)
        assert e <= TOL, (e, rel, cos)
