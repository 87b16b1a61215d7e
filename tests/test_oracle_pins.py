"""Pins for the CPU oracle: each oracle step is checked against something other
than itself -- a library routine (numpy's fp16 cast, transformers' RoPE,
scipy's Hadamard matrix, torch fp64 attention), a closed form, an invariant
the method relies on, or brute force on tiny inputs.

Passages: "RotateAttention: RoPE-Aware Rotation and Range Rectification for
INT4 Quantized Attention in Video Generation", abstract (3D RoPE,
RoPE-aware rotation, INT4 FlashAttention, range-optimised P quantisation with
fixed scale and zero-point, FP16 fallback).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from video_dit_b200 import synth

from codes import unpack


# ------------------------------------------------------------ fp16 casts ---

def test_half_to_float_exhaustive():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float32)
    got = np.array([oracle.half_to_float(int(b)) for b in bits], np.float32)
    finite = np.isfinite(ref)
    assert np.array_equal(got[finite].view(np.uint32), ref[finite].view(np.uint32))
    assert np.all(np.isnan(got[np.isnan(ref)]))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_float_to_half_rne_against_numpy():
    rng = np.random.default_rng(0)
    h = np.arange(0, 0x7bff, 7, dtype=np.uint16).view(np.float16).astype(np.float32)
    # exact halves, midpoints between neighbours (ties), 1 fp32 ulp either side, randoms
    nxt = np.nextafter(h.astype(np.float16), np.float16(np.inf)).astype(np.float32)
    mid = ((h.astype(np.float64) + nxt.astype(np.float64)) / 2).astype(np.float32)
    xs = np.concatenate([h, mid, np.nextafter(mid, np.float32(0)), np.nextafter(mid, np.float32(1e9)),
                         rng.standard_normal(20000).astype(np.float32) * 30,
                         rng.standard_normal(2000).astype(np.float32) * 1e-5,
                         np.float32([65504, 65519.9, 65520, 1e6, 2.0 ** -25, 2.0 ** -24 * 1.5])])
    xs = np.concatenate([xs, -xs])
    with np.errstate(over="ignore"):
        ref = xs.astype(np.float16).view(np.uint16)
    got = np.array([oracle.float_to_half(float(x)) for x in xs], np.uint16)
    assert np.array_equal(got, ref)


# ------------------------------------------------------------------ RoPE ---

def _hf_rope_axis(d_a, npos, theta):
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding
    cfg = LlamaConfig(hidden_size=d_a * 2, num_attention_heads=2, head_dim=d_a, rope_theta=theta)
    emb = LlamaRotaryEmbedding(cfg)
    pos = torch.arange(npos)[None]
    cos, sin = emb(torch.zeros(1, npos, d_a, dtype=torch.float64), pos)
    return cos[0].numpy(), sin[0].numpy()          # [npos, d_a], half-split layout


@pytest.mark.parametrize("rope_dim,grid", [((16, 24, 24), (4, 8, 8)), ((44, 42, 42), (21, 30, 52)),
                                           ((16, 56, 56), (33, 34, 60))])
def test_rope_tables_match_transformers(rope_dim, grid):
    c, s = oracle.rope_tables(grid, rope_dim)
    off = 0
    for a in range(3):
        half = rope_dim[a] // 2
        hc, hs = _hf_rope_axis(rope_dim[a], grid[a], 10000.0)
        oc = c[off: off + grid[a] * half].reshape(grid[a], half)
        os_ = s[off: off + grid[a] * half].reshape(grid[a], half)
        # transformers' inv_freq is fp32, so angles agree to ~pos * 1e-7
        assert np.abs(oc - hc[:, :half]).max() < 2e-5
        assert np.abs(os_ - hs[:, :half]).max() < 2e-5
        off += grid[a] * half


def test_rope_row_matches_transformers_apply():
    """Interleaved pairs (2i, 2i+1) of the oracle == transformers' half-split
    rotate_half after the channel permutation (i, i + d_a/2) <- (2i, 2i+1)."""
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    rope_dim, grid = (44, 42, 42), (21, 30, 52)
    rng = np.random.default_rng(1)
    for n in [0, 1, 52, 1561, 32759, 17 * 1560 + 29 * 52 + 51]:
        x = rng.standard_normal(128).astype(np.float32)
        y = oracle.rope_rotate_row(x, n, grid, rope_dim, (1, 1, 1), rotate=False)
        pos = (n // (30 * 52), (n // 52) % 30, n % 52)
        off = 0
        for a in range(3):
            d_a = rope_dim[a]
            hc, hs = _hf_rope_axis(d_a, grid[a], 10000.0)
            part = x[off: off + d_a].astype(np.float64)
            hf_in = np.concatenate([part[0::2], part[1::2]])
            t = torch.from_numpy(hf_in)[None, None, None]
            cos = torch.from_numpy(hc[pos[a]])[None, None]
            sin = torch.from_numpy(hs[pos[a]])[None, None]
            out, _ = apply_rotary_pos_emb(t, t, cos, sin)
            out = out[0, 0, 0].numpy()
            want = np.empty(d_a)
            want[0::2], want[1::2] = out[: d_a // 2], out[d_a // 2:]
            assert np.abs(y[off: off + d_a] - want).max() < 1e-4 * (1 + np.abs(want).max())
            off += d_a


@pytest.mark.parametrize("rope_dim,grid", [((44, 42, 42), (21, 30, 52)), ((16, 56, 56), (33, 34, 60)),
                                           ((16, 24, 24), (4, 8, 8))])
def test_rope_rounding_order_bit_exact(rope_dim, grid):
    """The RoPE arithmetic defines the quantiser's inputs bit for bit: pair
    (2i, 2i+1) of partition a at position p becomes
    y0 = RN(RN(x0 c) - RN(x1 s)), y1 = RN(RN(x0 s) + RN(x1 c)), every product
    and sum a separate fp32 rounding (no fused multiply-add), c / s the fp32
    table entries.  numpy float32 scalars round each operation once, in the
    order written here, so a contracted FMA or a swapped operand in the oracle
    changes some of these bits."""
    c_tab, s_tab = oracle.rope_tables(grid, rope_dim)
    rng = np.random.default_rng(11)
    d = sum(rope_dim)
    T, Hh, W = grid
    toks = [0, 1, W, Hh * W, T * Hh * W - 1] + list(rng.integers(0, T * Hh * W, 40))
    halves = [r // 2 for r in rope_dim]
    toff = [0, T * halves[0], T * halves[0] + Hh * halves[1]]
    fused_differs = 0
    for n in toks:
        n = int(n)
        pos = (n // (Hh * W), (n // W) % Hh, n % W)
        x = (rng.standard_normal(d) * rng.choice([1.0, 15.0, 300.0], d)).astype(np.float32)
        got = oracle.rope_rotate_row(x, n, grid, rope_dim, (1, 1, 1), rotate=False)
        want = np.empty(d, np.float32)
        off = 0
        for a in range(3):
            for i in range(halves[a]):
                c = np.float32(c_tab[toff[a] + pos[a] * halves[a] + i])
                s_ = np.float32(s_tab[toff[a] + pos[a] * halves[a] + i])
                x0, x1 = np.float32(x[off + 2 * i]), np.float32(x[off + 2 * i + 1])
                want[off + 2 * i] = np.float32(np.float32(x0 * c) - np.float32(x1 * s_))
                want[off + 2 * i + 1] = np.float32(np.float32(x0 * s_) + np.float32(x1 * c))
                # the contracted form fma(x0, c, -RN(x1 s)): the fp32 product is
                # exact in double, so one rounding of the double difference
                fz = np.float32(np.float64(x0) * np.float64(c) - np.float64(np.float32(x1 * s_)))
                fused_differs += int(fz != want[off + 2 * i])
            off += rope_dim[a]
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), n
    # the check can tell: a contracted multiply-add gives other bits on these rows
    assert fused_differs > 0


def test_unquantised_reference_matches_torch_sdpa_float64():
    """oracle.attn_ref (the reference of the cosine report): fp32 RoPE rows,
    no rotation, no rounding to fp16, softmax attention in double; against
    torch's float64 scaled_dot_product_attention on the same RoPE'd rows."""
    w = synth.scaled(synth.WORKLOADS["wan480"], "ref_pin", H=2, grid=(2, 5, 9))      # N = 90
    q, k, v = synth.make_inputs(w, seed=4)
    sm = float(np.float32(1 / math.sqrt(w.d)))
    for h in range(w.H):
        qr = np.stack([oracle.rope_rotate_row(q[0, h, n].astype(np.float32), n, w.grid, w.rope_dim,
                                              w.had_block, rotate=False) for n in range(w.N)])
        kr = np.stack([oracle.rope_rotate_row(k[0, h, n].astype(np.float32), n, w.grid, w.rope_dim,
                                              w.had_block, rotate=False) for n in range(w.N)])
        vv = v[0, h].astype(np.float64)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qr.astype(np.float64))[None], torch.from_numpy(kr.astype(np.float64))[None],
            torch.from_numpy(vv)[None], scale=sm)[0].numpy()
        got = oracle.attn_ref(q, k, v, w.grid, w.rope_dim, sm, 0, h, 0, w.N)
        assert np.abs(got - ref).max() <= 1e-12 * max(1.0, np.abs(ref).max())


def test_rope_identity_at_origin_and_relative_position():
    rope_dim, grid = (16, 24, 24), (4, 8, 8)
    rng = np.random.default_rng(2)
    q = rng.standard_normal(64).astype(np.float32)
    k = rng.standard_normal(64).astype(np.float32)
    y = oracle.rope_rotate_row(q, 0, grid, rope_dim, (1, 1, 1), rotate=False)
    assert np.array_equal(y, q)

    def tok(t, h, w):
        return (t * grid[1] + h) * grid[2] + w
    # (t,h,w) pairs and a shift; dot products depend only on the offset
    for (p1, p2, sh) in [((0, 0, 0), (1, 3, 5), (2, 4, 2)), ((1, 7, 2), (0, 1, 7), (1, 0, 0)),
                         ((0, 2, 6), (3, 0, 0), (0, 3, 1))]:
        a = np.dot(oracle.rope_rotate_row(q, tok(*p1), grid, rope_dim, (1, 1, 1), rotate=False),
                   oracle.rope_rotate_row(k, tok(*p2), grid, rope_dim, (1, 1, 1), rotate=False))
        s1 = tuple(x + s for x, s in zip(p1, sh))
        s2 = tuple(x + s for x, s in zip(p2, sh))
        b = np.dot(oracle.rope_rotate_row(q, tok(*s1), grid, rope_dim, (1, 1, 1), rotate=False),
                   oracle.rope_rotate_row(k, tok(*s2), grid, rope_dim, (1, 1, 1), rotate=False))
        assert abs(a - b) < 1e-4 * (1 + abs(a))


def _pair_rotate(y: np.ndarray, rope_dim, phase) -> np.ndarray:
    """Rotate every RoPE pair (2i, 2i+1) of partition a by phase[a], in double."""
    out = y.astype(np.float64).copy()
    c0 = 0
    for a, da in enumerate(rope_dim):
        ph = float(np.float32(phase[a]))
        c, s = math.cos(ph), math.sin(ph)
        for i in range(c0, c0 + da, 2):
            x0, x1 = out[i], out[i + 1]
            out[i], out[i + 1] = c * x0 - s * x1, s * x0 + c * x1
        c0 += da
    return out


@pytest.mark.parametrize("phase", [(0.3, math.pi / 4, -math.pi / 4), (-2.5, 1.0, 3.0)])
def test_merged_rotation_is_rope_then_pair_rotation(phase):
    """The phase in the tables equals RoPE followed by a fixed rotation of each
    pair (closed form in double; the tables' fp32 rounding is the only gap), is
    the pure pair rotation at position 0, and cancels in q.k (same phase on Q
    and K) up to that rounding."""
    rope_dim, grid = (44, 42, 42), (3, 5, 7)
    rng = np.random.default_rng(13)
    q = rng.standard_normal(128).astype(np.float32)
    k = rng.standard_normal(128).astype(np.float32)
    for n in (0, 17, 104):
        yp = oracle.rope_rotate_row(q, n, grid, rope_dim, (1, 1, 1), rotate=False, phase=phase)
        y0 = oracle.rope_rotate_row(q, n, grid, rope_dim, (1, 1, 1), rotate=False)
        assert np.abs(yp - _pair_rotate(y0, rope_dim, phase)).max() < 1e-5 * np.abs(q).max()
    y = oracle.rope_rotate_row(q, 0, grid, rope_dim, (1, 1, 1), rotate=False, phase=phase)
    assert np.abs(y - _pair_rotate(q, rope_dim, phase)).max() < 1e-6 * np.abs(q).max()
    for n1, n2 in ((0, 0), (5, 77), (104, 3)):
        a = np.dot(oracle.rope_rotate_row(q, n1, grid, rope_dim, (1, 1, 1), rotate=False, phase=phase).astype(np.float64),
                   oracle.rope_rotate_row(k, n2, grid, rope_dim, (1, 1, 1), rotate=False, phase=phase))
        b = np.dot(oracle.rope_rotate_row(q, n1, grid, rope_dim, (1, 1, 1), rotate=False).astype(np.float64),
                   oracle.rope_rotate_row(k, n2, grid, rope_dim, (1, 1, 1), rotate=False))
        assert abs(a - b) < 1e-4 * (1 + abs(b))


# -------------------------------------------------------------- rotation ---

@pytest.mark.parametrize("rope_dim,had", [((16, 24, 24), (16, 8, 8)), ((44, 42, 42), (4, 2, 2)),
                                          ((16, 56, 56), (16, 8, 8)), ((44, 42, 42), (1, 1, 1))])
def test_rotation_is_blockdiag_sylvester_hadamard(rope_dim, had):
    from scipy.linalg import block_diag, hadamard
    d = sum(rope_dim)
    M = np.stack([oracle.rope_rotate_row(np.eye(d, dtype=np.float32)[j], 0, (1, 1, 1), rope_dim, had,
                                         rope=False) for j in range(d)], axis=1)
    blocks = []
    for a in range(3):
        b = had[a]
        blocks += [hadamard(b) / math.sqrt(b)] * (rope_dim[a] // b)
    want = block_diag(*blocks)
    assert np.abs(M - want).max() <= 1e-7
    assert np.abs(M @ M.T - np.eye(d)).max() < 1e-6


@pytest.mark.parametrize("n", [12, 20, 24, 28, 36, 40, 44, 48, 56, 60])
def test_nonpow2_hadamard_is_hadamard(n):
    """H H^T = n I exactly, entries +-1 (the definition of a Hadamard matrix)."""
    h = oracle.hadamard(n)
    assert h is not None
    assert set(np.unique(h).tolist()) == {-1, 1}
    assert np.array_equal(h.astype(np.int64) @ h.T.astype(np.int64), n * np.eye(n, dtype=np.int64))


@pytest.mark.parametrize("n", [6, 10, 14, 18, 22, 52])
def test_nonpow2_hadamard_unsupported_orders(n):
    # 2 mod 4 orders > 2 admit no Hadamard matrix; 52 is none of the three constructions
    assert oracle.hadamard(n) is None


@pytest.mark.parametrize("rope_dim,had", [((44, 42, 42), (44, 2, 2)), ((16, 56, 56), (16, 56, 56)),
                                          ((24, 20, 20), (12, 20, 20))])
def test_dense_rotation_is_normalised_hadamard_and_keeps_qk(rope_dim, had):
    """A non-power-of-two block is the dense product (H / sqrt(b)) x (checked in
    double against the matrix), and q.k is unchanged by it."""
    grid = (2, 3, 5)
    d = sum(rope_dim)
    rng = np.random.default_rng(17)
    q = rng.standard_normal(d).astype(np.float32)
    k = rng.standard_normal(d).astype(np.float32)
    yq = oracle.rope_rotate_row(q, 7, grid, rope_dim, had)
    y0 = oracle.rope_rotate_row(q, 7, grid, rope_dim, (1, 1, 1), rotate=True)
    # the expected rotation, block by block, in double
    want = y0.astype(np.float64).copy()
    c0 = 0
    for a, (da, b) in enumerate(zip(rope_dim, had)):
        if b > 1:
            m = oracle.hadamard(b) if b & (b - 1) else None
            if m is None:
                from scipy.linalg import hadamard as sylvester
                m = sylvester(b)
            for blk in range(c0, c0 + da, b):
                want[blk:blk + b] = (m.astype(np.float64) @ want[blk:blk + b]) / math.sqrt(b)
        c0 += da
    assert np.abs(yq - want).max() < 1e-5 * np.abs(want).max()
    yk = oracle.rope_rotate_row(k, 11, grid, rope_dim, had)
    zk = oracle.rope_rotate_row(k, 11, grid, rope_dim, (1, 1, 1), rotate=True)
    a = float(np.dot(yq.astype(np.float64), yk))
    b = float(np.dot(y0.astype(np.float64), zk))
    assert abs(a - b) < 1e-4 * (1 + abs(b))


def test_rotation_preserves_qk():
    rope_dim, had = (44, 42, 42), (4, 2, 2)
    rng = np.random.default_rng(3)
    for _ in range(20):
        q = (rng.standard_normal(128) * np.where(rng.random(128) < 0.05, 15, 1)).astype(np.float32)
        k = rng.standard_normal(128).astype(np.float32)
        rq = oracle.rope_rotate_row(q, 0, (1, 1, 1), rope_dim, had, rope=False)
        rk = oracle.rope_rotate_row(k, 0, (1, 1, 1), rope_dim, had, rope=False)
        ref = np.dot(q.astype(np.float64), k.astype(np.float64))
        assert abs(np.dot(rq.astype(np.float64), rk.astype(np.float64)) - ref) < 1e-5 * (
            np.abs(q).sum() * np.abs(k).max())


# ------------------------------------------------------------- quantiser ---

@pytest.mark.parametrize("amax", [1.0, 0.3, 7.0, 42.123, 65504.0, 3.1e-3])
def test_quantiser_exhaustive_fp16(amax):
    ys = np.arange(65536, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float32)
    ys = ys[np.isfinite(ys) & (np.abs(ys) <= np.float32(amax))]
    scale, inv = oracle.quant_params(amax)
    assert scale == np.float32(amax) / np.float32(7) and inv == np.float32(7) / np.float32(amax)
    c = oracle.quant_codes(ys, inv).astype(np.int64)
    assert c.min() >= -7 and c.max() <= 7
    # numpy's IEEE fp32 multiply and round-half-even give the same codes
    assert np.array_equal(c, np.clip(np.rint(ys * np.float32(inv)), -7, 7).astype(np.int64))
    err = np.abs(ys.astype(np.float64) - c * np.float64(scale))
    assert err.max() <= np.float64(scale) / 2 * (1 + 2.0 ** -20)
    order = np.argsort(ys, kind="stable")
    assert np.all(np.diff(c[order]) >= 0)                     # monotone
    assert oracle.quant_code(amax, inv) == 7 and oracle.quant_code(-amax, inv) == -7
    assert np.array_equal(oracle.quant_codes(-ys, inv), -oracle.quant_codes(ys, inv))


def test_quantiser_zero_block():
    assert oracle.quant_params(0.0) == (0.0, 0.0)
    assert oracle.quant_code(0.0, 0.0) == 0


def test_code_packing_layout():
    rng = np.random.default_rng(5)
    v = rng.integers(-7, 8, size=(37, 64)).astype(np.int32)
    packed = oracle.pack_codes(v)
    assert packed.shape == (37, 32)
    assert np.array_equal(unpack(packed), v)
    # spot values: e0 = -3, e4 = 5 -> byte 0 = 0x5B; zero stays 0000
    w = np.zeros((1, 8), np.int32)
    w[0, 0], w[0, 4], w[0, 7] = -3, 5, -7
    assert list(oracle.pack_codes(w)[0]) == [0x5B, 0x00, 0x00, 0xF0]
    assert [oracle.lib().oracle_code_at(oracle._p(oracle.pack_codes(w)[0].copy()), i) for i in range(8)] == \
        [-3, 0, 0, 0, 5, 0, 0, -7]


# --------------------------------------------------------------- P codes ---

def _thresholds():
    """tau_k: the smallest fp32 d with RNE(15 * 2^d) >= k, from mpmath at 60 digits."""
    import mpmath
    mpmath.mp.dps = 60
    taus = {}
    for k in range(1, 16):
        t = mpmath.log((mpmath.mpf(k) - mpmath.mpf("0.5")) / 15, 2)
        f = np.float32(float(t))
        while mpmath.mpf(float(f)) < t:
            f = np.nextafter(f, np.float32(1))
        while mpmath.mpf(float(np.nextafter(f, np.float32(-10)))) >= t:
            f = np.nextafter(f, np.float32(-10))
        taus[k] = f
    return taus


def test_pcode_thresholds():
    taus = _thresholds()
    assert taus[8] == np.float32(-1.0)          # 15 * 2^-1 = 7.5 is the only tie: RNE -> 8
    for k, t in taus.items():
        assert oracle.pcode(float(t)) == k, (k, t)
        assert oracle.pcode(float(np.nextafter(t, np.float32(-10)))) == k - 1, (k, t)
    assert oracle.pcode(0.0) == 15
    assert oracle.pcode(-0.0) == 15
    assert oracle.pcode(-200.0) == 0
    assert oracle.pcode(3e-8) == 15


def test_pcode_dense_sample_matches_threshold_form():
    taus = _thresholds()
    tau = np.array([taus[k] for k in range(1, 16)], np.float32)
    rng = np.random.default_rng(4)
    d = np.concatenate([rng.uniform(-6, 0, 2_000_000).astype(np.float32),
                        (tau[:, None] + np.arange(-64, 65)[None, :] * np.float32(2 ** -22)).ravel()])
    d = d[d <= 0]
    u = oracle.pcode_array(d)
    want = np.searchsorted(tau, d, side="right")             # #{k: tau_k <= d}
    assert np.array_equal(u.astype(np.int64), want)


def _max_key_codes(lo: float, hi: float, n: int = 20000, seed: int = 12):
    """P code of the key that sets the running max, m = RN(S c), for n random
    (S_int, c) with |S c| in [lo, hi): d = RN(S c - m) (the one rounding of the
    fma; S c - m is exact in double)."""
    rng = np.random.default_rng(seed)
    s_int = rng.integers(1, 49 * 128, n).astype(np.float64)
    x = np.exp(rng.uniform(np.log(lo), np.log(hi), n))
    c = (x / s_int).astype(np.float32).astype(np.float64)
    m = (s_int * c).astype(np.float32).astype(np.float64)
    d = (s_int * c - m).astype(np.float32)
    return oracle.pcode_array(d)


def test_max_key_keeps_code_15_below_2_pow_20():
    """The row sum is at least 15 (the key that sets the max has code 15) while
    the logits stay below 2^20: there the rounding of m moves that key's
    exponent by at most half an ulp of m, <= 2^-5, well inside log2(14.5/15).
    Beyond 2^21 the half ulp exceeds it and the code can drop."""
    assert (_max_key_codes(1e-3, 2.0 ** 20) == 15).all()
    assert math.log2(14.5 / 15) < -(2.0 ** -5)
    assert (_max_key_codes(2.0 ** 21, 2.0 ** 24) < 15).any()


# ------------------------------------------------------ whole pipeline ---

def _tiny(**kw):
    w = synth.WORKLOADS["tiny"]
    return synth.scaled(w, "tiny_pin", **kw) if kw else w


def test_prepare_codes_reconstruct_rotated_values():
    w = _tiny()
    q, k, v = synth.make_inputs(w)
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    for name, src in (("q", q), ("k", k)):
        codes = unpack(p[f"{name}_codes"][0, 1]).astype(np.float64)
        scale = np.repeat(p[f"{name}_scale"][0, 1], 64).astype(np.float64)
        for n in range(0, w.N, 37):
            y = oracle.rope_rotate_row(src[0, 1, n].astype(np.float32), n, w.grid, w.rope_dim, w.had_block)
            assert np.abs(codes[n] * scale[n] - y).max() <= scale[n] / 2 * (1 + 1e-6)
        for j in range(w.N // 64):
            assert np.abs(codes[j * 64:(j + 1) * 64]).max() == 7
    vc = unpack(p["v_codes"][0, 0]).astype(np.float64)       # [blk, d, 64]
    vs = p["v_scale"][0, 0].astype(np.float64)                          # [blk, d]
    deq = (vc * vs[:, :, None]).transpose(0, 2, 1).reshape(-1, w.d)
    vv = v[0, 0].astype(np.float64)
    assert np.all(np.abs(deq - vv) <= np.repeat(vs, 64, axis=0) / 2 * (1 + 1e-6))


def test_integer_scores_brute_force():
    w = _tiny()
    q, k, v = synth.make_inputs(w)
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    _, s, _ = oracle.attn_int4(p, w.N, 1 / math.sqrt(w.d), 0, 1, 0, w.N, dump=True)
    qc = unpack(p["q_codes"][0, 1]).astype(np.int64)
    kc = unpack(p["k_codes"][0, 1]).astype(np.int64)
    assert np.array_equal(s, qc @ kc.T)


def test_pcodes_span_full_range_and_offset_identity():
    w = _tiny()
    q, k, v = synth.make_inputs(w)
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    hist = np.zeros(16, np.int64)
    for h in range(w.H):
        _, _, u = oracle.attn_int4(p, w.N, 1 / math.sqrt(w.d), 0, h, 0, w.N, dump=True)
        hist += np.bincount(u.ravel(), minlength=16)
        vc = unpack(p["v_codes"][0, h]).astype(np.int64)    # [blk, d, 64]
        for j in range(w.N // 64):
            uj = u[:, j * 64:(j + 1) * 64].astype(np.int64)
            lhs = uj @ vc[j].T
            rhs = (uj - 8) @ vc[j].T + 8 * vc[j].sum(axis=1)[None, :]
            assert np.array_equal(lhs, rhs)
    assert np.all(hist > 0), hist          # unsigned codes use all 16 levels


def test_online_and_closed_forms_agree():
    w = synth.scaled(synth.WORKLOADS["wan480"], "mini", H=1, grid=(2, 5, 13))     # N = 130: ragged
    q, k, v = synth.make_inputs(w)
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    a = oracle.attn_int4(p, w.N, 1 / math.sqrt(w.d), 0, 0, 0, w.N, online=False)
    b = oracle.attn_int4(p, w.N, 1 / math.sqrt(w.d), 0, 0, 0, w.N, online=True)
    assert np.abs(a - b).max() < 1e-12 * (1 + np.abs(a).max())


def test_uniform_attention_when_scores_vanish():
    """Q = 0 -> every score is 0 -> every P code is 15 -> the output is the
    mean of the dequantised V rows."""
    w = synth.scaled(synth.WORKLOADS["wan480"], "zeroq", H=1, grid=(1, 5, 20))     # N = 100
    q, k, v = synth.make_inputs(w)
    q[:] = 0
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    out, _, u = oracle.attn_int4(p, w.N, 1 / math.sqrt(w.d), 0, 0, 0, w.N, dump=True)
    assert np.all(u == 15)
    vc = unpack(p["v_codes"][0, 0]).astype(np.float64)
    deq = (vc * p["v_scale"][0, 0].astype(np.float64)[:, :, None]).transpose(0, 2, 1).reshape(-1, w.d)
    assert np.abs(out - deq[: w.N].mean(axis=0)[None]).max() < 1e-12


def test_dominant_key_selects_its_value_row():
    w = synth.scaled(synth.WORKLOADS["wan480"], "dom", H=1, grid=(1, 4, 32), qk_outliers=(0, 0, 0))
    q, k, v = synth.make_inputs(w)
    j = 10       # in the first key group: later groups are all coded against its max
    k[0, 0, j] = np.float16(0)
    k[0, 0, j, ::3] = np.float16(6)
    q[0, 0, :] = np.float16(0)
    q[0, 0, :, ::3] = np.float16(6)        # RoPE is position dependent: keep only row j's own token
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    out, s, u = oracle.attn_int4(p, w.N, 1 / math.sqrt(w.d), 0, 0, j, 1, dump=True)
    assert u[0, j] == 15 and u[0].sum() == 15
    vc = unpack(p["v_codes"][0, 0]).astype(np.float64)
    row = vc[j // 64, :, j % 64] * p["v_scale"][0, 0, j // 64].astype(np.float64)
    assert np.abs(out[0] - row).max() < 1e-12


def test_single_group_is_global_max():
    """group >= N: every P code is taken against the final row max."""
    w = synth.scaled(synth.WORKLOADS["wan480"], "glob", H=1, grid=(2, 5, 13))
    q, k, v = synth.make_inputs(w)
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    out, s, u = oracle.attn_int4(p, w.N, 1 / math.sqrt(w.d), 0, 0, 0, w.N, group=1 << 20, dump=True)
    assert np.all(u.max(axis=1) == 15)
    kappa = np.float32(np.float64(np.float32(1 / math.sqrt(w.d))) * 1.4426950408889634)
    qs = np.repeat(p["q_scale"][0, 0], 64)[: w.N]
    ks = np.repeat(p["k_scale"][0, 0], 64)[: w.N]
    c = (qs[:, None] * ks[None, :]).astype(np.float32) * kappa
    x = s.astype(np.float32) * c
    M = x.max(axis=1, keepdims=True)
    dd = (s.astype(np.float64) * c.astype(np.float64) - M).astype(np.float32)  # one rounding
    assert np.array_equal(u, oracle.pcode_array(dd))
    vc = unpack(p["v_codes"][0, 0]).astype(np.float64)
    deq = (vc * p["v_scale"][0, 0].astype(np.float64)[:, :, None]).transpose(0, 2, 1).reshape(-1, w.d)
    want = (u.astype(np.float64) @ deq[: w.N]) / u.sum(axis=1, keepdims=True)
    assert np.abs(out - want).max() < 1e-12


def test_max_group_128_is_global_max_below_129_keys():
    """With N <= 128 keys a 128-key group holds every key, so the codes and the
    output equal those of the single global group, bit for bit."""
    w = synth.scaled(synth.WORKLOADS["wan480"], "g128", H=1, grid=(1, 2, 50))   # N = 100
    q, k, v = synth.make_inputs(w)
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    sm = 1 / math.sqrt(w.d)
    o128, s128, u128 = oracle.attn_int4(p, w.N, sm, 0, 0, 0, w.N, group=128, dump=True)
    og, sg, ug = oracle.attn_int4(p, w.N, sm, 0, 0, 0, w.N, group=1 << 20, dump=True)
    assert np.array_equal(u128, ug) and np.array_equal(s128, sg)
    assert np.array_equal(o128, og)
    # and the 64-key reading differs on these rows (the pin can tell them apart)
    _, _, u64 = oracle.attn_int4(p, w.N, sm, 0, 0, 0, w.N, group=64, dump=True)
    assert not np.array_equal(u64, ug)


def test_fp16_path_matches_torch_sdpa_float64():
    w = synth.scaled(synth.WORKLOADS["wan480"], "f16", H=2, grid=(2, 5, 13))
    q, k, v = synth.make_inputs(w)
    flags = np.ones(w.H, np.uint8)
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block, flags=flags)
    qr = torch.from_numpy(p["q_rope"].view(np.float16).astype(np.float64))
    kr = torch.from_numpy(p["k_rope"].view(np.float16).astype(np.float64))
    vv = torch.from_numpy(v.astype(np.float64))
    sm = float(np.float32(1 / math.sqrt(w.d)))       # the oracle takes sm_scale as fp32
    ref = torch.nn.functional.scaled_dot_product_attention(qr, kr, vv, scale=sm).numpy()
    for h in range(w.H):
        out = oracle.attn_fp16(p["q_rope"], p["k_rope"], v, 1 / math.sqrt(w.d), 0, h, 0, w.N)
        assert np.abs(out - ref[0, h]).max() < 1e-12
    # q_rope is the fp16 rounding of the RoPE'd row
    for n in (0, 5, 129):
        y = oracle.rope_rotate_row(q[0, 1, n].astype(np.float32), n, w.grid, w.rope_dim, w.had_block,
                                   rotate=False)
        assert np.array_equal(p["q_rope"][0, 1, n], y.astype(np.float16).view(np.uint16))


def test_int4_close_to_unquantised_attention_on_plain_gaussians():
    w = synth.scaled(synth.WORKLOADS["tiny"], "plain", qk_outliers=(0, 0, 0))
    q, k, v = synth.make_inputs(w)
    p = oracle.prepare(q, k, v, w.grid, w.rope_dim, w.had_block)
    out = oracle.attn_int4(p, w.N, 1 / math.sqrt(w.d), 0, 0, 0, w.N)
    ref = oracle.attn_ref(q, k, v, w.grid, w.rope_dim, 1 / math.sqrt(w.d), 0, 0, 0, w.N)
    cos = (out * ref).sum(1) / np.linalg.norm(out, axis=1) / np.linalg.norm(ref, axis=1)
    assert cos.mean() > 0.93 and cos.min() > 0.75


# ------------------------------------------------- numerics options (R1, G = 128)

def _unit_c_scales(sm_scale):
    """(sq, sk) with c = RN(RN(sq sk) kappa) == 1 exactly, kappa = RN(sm_scale log2 e)."""
    kappa = np.float32(np.float64(np.float32(sm_scale)) * 1.4426950408889634074)
    base = np.float32(1.0) / kappa
    for step in range(-64, 65):
        sk = np.array([base], np.float32).view(np.int32).__add__(np.int32(step)).view(np.float32)[0]
        if np.float32(np.float32(np.float32(1.0) * sk) * kappa) == np.float32(1.0):
            return np.float32(1.0), sk
    raise AssertionError("no key scale gives c = 1")


def _hand_prep(q_rows, k_rows, v_blocks, sq, sk, d=8):
    """A one-head prepared problem from explicit codes: q_rows [n, d], k_rows
    [N, d] (codes in [-7, 7]), v_blocks [nblk, d, 64]; every scale is 1 except
    the Q / K block scales sq, sk."""
    N = len(k_rows)
    nblk = (N + 63) // 64
    npad = nblk * 64
    q = np.zeros((npad, d), np.int32)
    q[:len(q_rows)] = q_rows
    k = np.zeros((npad, d), np.int32)
    k[:N] = k_rows
    return {"q_codes": oracle.pack_codes(q)[None, None], "k_codes": oracle.pack_codes(k)[None, None],
            "q_scale": np.full((1, 1, nblk), sq, np.float32), "k_scale": np.full((1, 1, nblk), sk, np.float32),
            "v_codes": oracle.pack_codes(np.asarray(v_blocks, np.int32))[None, None],
            "v_scale": np.ones((1, 1, nblk, d), np.float32)}


def test_row_sum_readings_closed_form():
    """Two keys with scores x = 1 and x = 0 (c = 1): exponents d = 0 and -1,
    codes 15 and 8 (7.5 rounds to even), unquantised 15 * 2^d = 15 and 7.5.
    R2 divides by the code sum 23, R1 by 22.5; the numerator is
    15 v0 + 8 v1 either way."""
    sm = 0.125
    sq, sk = _unit_c_scales(sm)
    qr = np.zeros((1, 8), np.int32)
    qr[0, 0] = 1
    kr = np.zeros((2, 8), np.int32)
    kr[0, 0] = 1                                   # S = 1 -> x = 1 = the max
    vb = np.zeros((1, 8, 64), np.int32)
    vb[0, :, 0] = [1, -2, 3, -4, 5, -6, 7, 0]      # key 0
    vb[0, :, 1] = [7, 6, 5, 4, 3, 2, 1, -1]        # key 1
    prep = _hand_prep(qr, kr, vb, sq, sk)
    o2, s, u = oracle.attn_int4(prep, 2, sm, 0, 0, 0, 1, dump=True)
    o1 = oracle.attn_int4(prep, 2, sm, 0, 0, 0, 1, rowsum=1)
    assert s.tolist() == [[1, 0]] and u.tolist() == [[15, 8]]
    num = 15.0 * vb[0, :, 0] + 8.0 * vb[0, :, 1]
    assert np.abs(o2[0] - num / 23.0).max() < 1e-15
    assert np.abs(o1[0] - num / 22.5).max() < 1e-15


def test_max_group_128_closed_form():
    """Block 0: 64 keys with x = 0; block 1: key 64 with x = 1, the other 63
    with x = 0 (c = 1).  With 64-key groups block 0 is coded against its own
    max 0 (codes 15, weight 2^(0 - 1) = 1/2 at the end); with 128-key groups
    both blocks share the max 1 (block 0's codes drop to 8, weight 1).  V codes
    are 1 in block 0 and 2 in block 1 (all channels), every scale 1."""
    sm = 0.125
    sq, sk = _unit_c_scales(sm)
    qr = np.zeros((1, 8), np.int32)
    qr[0, 0] = 1
    kr = np.zeros((128, 8), np.int32)
    kr[64, 0] = 1
    vb = np.zeros((2, 8, 64), np.int32)
    vb[0] = 1
    vb[1] = 2
    prep = _hand_prep(qr, kr, vb, sq, sk)
    o64, _, u64 = oracle.attn_int4(prep, 128, sm, 0, 0, 0, 1, group=64, dump=True)
    o128, _, u128 = oracle.attn_int4(prep, 128, sm, 0, 0, 0, 1, group=128, dump=True)
    assert (u64[0, :64] == 15).all() and u64[0, 64] == 15 and (u64[0, 65:] == 8).all()
    assert (u128[0, :64] == 8).all() and u128[0, 64] == 15 and (u128[0, 65:] == 8).all()
    num64 = 0.5 * 64 * 15 * 1 + (15 + 63 * 8) * 2
    den64 = 0.5 * 64 * 15 + (15 + 63 * 8)
    num128 = 64 * 8 * 1 + (15 + 63 * 8) * 2
    den128 = 64 * 8 + (15 + 63 * 8)
    assert np.abs(o64[0] - num64 / den64).max() < 1e-14
    assert np.abs(o128[0] - num128 / den128).max() < 1e-14
    # R1 with 128-key groups: 15 * 2^-1 = 7.5 per block-0 key and per other block-1 key
    o128r1 = oracle.attn_int4(prep, 128, sm, 0, 0, 0, 1, group=128, rowsum=1)
    assert np.abs(o128r1[0] - num128 / (64 * 7.5 + 15 + 63 * 7.5)).max() < 1e-14


# ------------------------------------------------------------- QKV projection

def test_qkv_project_matches_numpy_and_exact_grid():
    """The oracle's projection against numpy (float64 matmul -> fp32 -> fp16)
    on general fp16 inputs, and against exact integer arithmetic on the grid
    inputs (k / 16 times j / 64: sums of multiples of 2^-10)."""
    w = synth.scaled(synth.WORKLOADS["wan480"], "qkv_pin", H=2, grid=(1, 3, 7))      # N = 21
    C = 128
    for exact in (False, True):
        x, wt = synth.make_qkv_inputs(w, C, seed=5, exact=exact)
        q, k, v = oracle.qkv_project(x, wt, w.H, w.d)
        full = x[0].astype(np.float64) @ wt.astype(np.float64).T                    # [N, 3 H d]
        want = full.astype(np.float32).astype(np.float16)
        for m, out in enumerate((q, k, v)):
            for h in range(w.H):
                cols = want[:, (m * w.H + h) * w.d:(m * w.H + h + 1) * w.d]
                assert np.array_equal(out[0, h].view(np.uint16), cols.view(np.uint16)), (exact, m, h)
        if exact:
            xi = np.round(x[0].astype(np.float64) * 16).astype(np.int64)
            wi = np.round(wt.astype(np.float64) * 64).astype(np.int64)
            ints = xi @ wi.T                                                           # exact, units 2^-10
            assert np.array_equal(ints.astype(np.float64) / 1024.0, full)
