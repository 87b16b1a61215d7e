"""Seeded synthetic inputs for the video-DiT attention workloads.

This module holds workload shapes and random draws only -- none of the
method's arithmetic -- so that the CUDA path's tests and the CPU oracle are
fed identical bytes.  The shapes follow the Wan-style 480p/720p and
HunyuanVideo-style latent grids (B, H, head_dim, 3D RoPE split, T x Hh x W
grid); the pages use no public dataset for this path, so Gaussian draws with
planted outlier channels (per RoPE partition, in Q and K) and outlier tokens
(in V) stand in for real activations.

Recipe (fixed; see the docstring of ``make_inputs``):
  * Q, K, V ~ N(0, 1) in fp32 [B, H, N, d], drawn in that order from a torch
    CPU generator seeded ``seed`` (default 0);
  * outlier channels: per RoPE partition and head, the first ``k`` of a
    ``randperm(d_a)`` for Q and then, independently, for K, from a generator
    seeded ``seed + 1``, offset to the partition (drawn independently: with
    coinciding channels at x15-x25 the logits reach tens of nats and the
    attention degenerates to an argmax);
  * V outlier tokens: per head, the first ceil(frac * N) of ``randperm(N)``
    from a generator seeded ``seed + 2``;
  * the scaled fp32 values are cast to fp16 (round to nearest even).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    rope_dim: Tuple[int, int, int]
    grid: Tuple[int, int, int]
    theta: float = 10000.0
    # outliers planted in Q and K: per partition a, `qk_outliers[a]` channels x `qk_scale`
    qk_outliers: Tuple[int, int, int] = (0, 0, 0)
    qk_scale: float = 1.0
    v_token_frac: float = 0.0
    v_token_scale: float = 1.0
    fp16_every: int = 0          # heads h with h % fp16_every == 0 take the FP16 fallback
    all_fp16: bool = False
    # rotation: Hadamard block per partition (None = the default block) and the
    # merged per-pair rotation angle added to every RoPE angle (0 = plain RoPE)
    had: Optional[Tuple[int, int, int]] = None
    rope_phase: Tuple[float, float, float] = (0.0, 0.0, 0.0)
    # numerics options of the INT4 path: key group of the running max, row-sum reading
    max_group: int = 64
    row_sum: int = 0

    @property
    def N(self) -> int:
        return self.grid[0] * self.grid[1] * self.grid[2]

    @property
    def had_block(self) -> Tuple[int, int, int]:
        if self.had is not None:
            return tuple(self.had)
        return tuple(default_had_block(r) for r in self.rope_dim)

    def flags(self) -> np.ndarray:
        f = np.zeros(self.H, np.uint8)
        if self.all_fp16:
            f[:] = 1
        elif self.fp16_every:
            f[:: self.fp16_every] = 1
        return f

    def ops(self) -> float:
        """Effective-op count of one attention call: 4 B H N^2 d."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d


def default_had_block(d_a: int) -> int:
    """Largest power of two dividing d_a, capped at 64 (Hadamard orders > 2
    are multiples of 4, so a partition of 42 takes blocks of 2)."""
    b = 1
    while d_a % (2 * b) == 0 and 2 * b <= 64:
        b *= 2
    return b


_WAN = dict(d=128, rope_dim=(44, 42, 42), qk_outliers=(4, 4, 4), qk_scale=15.0,
            v_token_frac=0.01, v_token_scale=8.0)

WORKLOADS = {
    "tiny": Workload("tiny", B=1, H=2, d=64, rope_dim=(16, 24, 24), grid=(4, 8, 8),
                     qk_outliers=(2, 2, 2), qk_scale=20.0),
    "wan480": Workload("wan480", B=1, H=40, grid=(21, 30, 52), **_WAN),
    "wan720": Workload("wan720", B=1, H=40, grid=(21, 45, 80), fp16_every=10, **_WAN),
    "hunyuan": Workload("hunyuan", B=1, H=24, d=128, rope_dim=(16, 56, 56), grid=(33, 34, 60),
                        qk_outliers=(4, 0, 0), qk_scale=25.0),
}
# the rotation variants on the full-size recipes: the whole 44-channel temporal partition
# as one Hadamard block (Paley I, q = 43) and the 56-channel ones (Paley II, q = 13, doubled)
WORKLOADS["wan480_h44"] = dataclasses.replace(WORKLOADS["wan480"], name="wan480_h44", had=(44, 2, 2))
WORKLOADS["hunyuan_h56"] = dataclasses.replace(WORKLOADS["hunyuan"], name="hunyuan_h56", had=(16, 56, 56))
# the P-code numerics variants on the 480p recipe: one max per 128 keys, and the R1 row sum
WORKLOADS["wan480_g128"] = dataclasses.replace(WORKLOADS["wan480"], name="wan480_g128", max_group=128)
WORKLOADS["wan480_r1"] = dataclasses.replace(WORKLOADS["wan480"], name="wan480_r1", row_sum=1)
for _F in (3, 6, 11, 21, 31):
    WORKLOADS[f"sweep{_F}"] = Workload(f"sweep{_F}", B=1, H=40, grid=(_F, 30, 52), **_WAN)
    WORKLOADS[f"sweep{_F}_fp16"] = Workload(f"sweep{_F}_fp16", B=1, H=40, grid=(_F, 30, 52),
                                           all_fp16=True, **_WAN)


def scaled(w: Workload, name: str, H: Optional[int] = None, grid=None, **kw) -> Workload:
    """A smaller copy of a workload with the same distributions (parity sizes)."""
    return dataclasses.replace(w, name=name, H=H or w.H, grid=tuple(grid or w.grid), **kw)


def make_inputs(w: Workload, seed: int = 0):
    """Q, K, V as fp16 numpy arrays [B, H, N, d] (recipe in the module docstring)."""
    B, H, N, d = w.B, w.H, w.N, w.d
    g0 = torch.Generator().manual_seed(seed)
    q = torch.randn((B, H, N, d), generator=g0, dtype=torch.float32)
    k = torch.randn((B, H, N, d), generator=g0, dtype=torch.float32)
    v = torch.randn((B, H, N, d), generator=g0, dtype=torch.float32)
    if any(w.qk_outliers):
        g1 = torch.Generator().manual_seed(seed + 1)
        mq = torch.ones((H, d), dtype=torch.float32)
        mk = torch.ones((H, d), dtype=torch.float32)
        off = 0
        for a in range(3):
            for h in range(H):
                for m in (mq, mk):
                    perm = torch.randperm(w.rope_dim[a], generator=g1)
                    m[h, perm[: w.qk_outliers[a]] + off] = w.qk_scale
            off += w.rope_dim[a]
        q.mul_(mq[None, :, None, :])
        k.mul_(mk[None, :, None, :])
    if w.v_token_frac > 0:
        g2 = torch.Generator().manual_seed(seed + 2)
        cnt = int(math.ceil(w.v_token_frac * N))
        for h in range(H):
            tok = torch.randperm(N, generator=g2)[:cnt]
            v[:, h, tok, :] *= w.v_token_scale
    return (q.to(torch.float16).numpy(), k.to(torch.float16).numpy(),
            v.to(torch.float16).numpy())


def make_qkv_inputs(w: Workload, C: int, seed: int = 0, exact: bool = True):
    """Inputs of the fused QKV projection: x fp16 [B, N, C] and the projection
    weights fp16 [3 H d, C] (rows of head h: Q at h d, K at H d + h d, V at
    2 H d + h d), Gaussian so that q, k, v come out about N(0, 1); the Q / K
    rows of the workload's outlier channels are scaled by its qk_scale.
    exact=True puts x on the grid k / 16 (|k| <= 128) and W on j / 64, so every
    product is a multiple of 2^-10 and every sum below 2^24 of those units:
    the fp32 accumulation is then exact in any order, and a projection's
    result does not depend on how it sums."""
    B, H, N, d = w.B, w.H, w.N, w.d
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((B, N, C), generator=g, dtype=torch.float64)
    wt = torch.randn((3 * H * d, C), generator=g, dtype=torch.float64) / math.sqrt(C)
    if any(w.qk_outliers):
        g1 = torch.Generator().manual_seed(seed + 1)
        off = 0
        for a in range(3):
            for h in range(H):
                for m in (0, 1):
                    perm = torch.randperm(w.rope_dim[a], generator=g1)
                    rows = m * H * d + h * d + off + perm[: w.qk_outliers[a]]
                    wt[rows] *= w.qk_scale
            off += w.rope_dim[a]
    if exact:
        x = torch.clamp(torch.round(x * 16), -128, 128) / 16
        wt = torch.round(wt * 64) / 64
        assert float(wt.abs().max()) * 64 <= 2048
        bound = C * 128 * float(wt.abs().max() * 64)          # |sum| in units of 2^-10
        assert bound < 2 ** 24, "inputs too wide for an exact fp32 accumulation"
    return x.to(torch.float16).numpy(), wt.to(torch.float16).numpy()
