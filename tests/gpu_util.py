"""Helpers shared by the GPU parity tests: run the library through the C ABI
on seeded numpy inputs and bring the results back as numpy arrays."""
import math

import numpy as np
import torch

from video_dit_b200 import synth


def lib():
    from video_dit_b200 import build
    build.build()
    from video_dit_b200 import rota_attn
    return rota_attn


def desc_of(w: synth.Workload):
    return lib().make_desc(w.B, w.H, w.d, w.grid, w.rope_dim, w.had_block, w.theta, rope_phase=w.rope_phase,
                        max_group=w.max_group, row_sum=w.row_sum)


def to_dev(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run(w: synth.Workload, q, k, v, flags=None, dump=None):
    """Prologue + attention on the GPU.  Returns (codes dict, out [B,H,N,d]
    float32, dump tuple or None).  dump=(b, h, r0, nr) adds the S / P dumps."""
    ra = lib()
    flags = np.zeros(w.H, np.uint8) if flags is None else np.asarray(flags, np.uint8)
    att = ra.RotaAttention(desc_of(w), need_fp16=bool(flags.any()))
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    out = torch.full((w.B, w.H, w.N, w.d), float("nan"), dtype=torch.float32, device="cuda")
    att.forward(qd, kd, vd, flags, out)
    dumped = None
    if dump is not None:
        b, h, r0, nr = dump
        s = torch.zeros((nr, w.N), dtype=torch.int32, device="cuda")
        p = torch.zeros((nr, w.N), dtype=torch.uint8, device="cuda")
        out2 = torch.empty_like(out)
        ra._check(ra.rota_attn_debug_dump_int4(att.desc, att.buffers, b, h, r0, nr, s, p, out2), "dump")
        dumped = (s.cpu().numpy(), p.cpu().numpy(), out2.cpu().numpy())
    st = ra.rota_attn_get_error()
    assert st == ra.ROTA_OK, ra.rota_attn_status_string(st)
    codes = {k_: (None if t is None else t.cpu().numpy()) for k_, t in att.codes().items()}
    if codes["q_rope"] is not None:
        codes["q_rope"] = codes["q_rope"].view(np.uint16)
        codes["k_rope"] = codes["k_rope"].view(np.uint16)
    return codes, out.cpu().numpy(), dumped


def kappa(head_dim: int) -> float:
    """The score scale's constant both sides use: RN(RN(1/sqrt(d)) * log2 e) from double."""
    s = np.float32(1.0 / math.sqrt(head_dim))
    return float(np.float32(np.float64(s) * 1.4426950408889634))


def sm_scale(w):
    return float(np.float32(1 / math.sqrt(w.d)))


def row_stats(got, ref):
    """max-abs error, max error relative to the row norm, min cosine."""
    err = np.abs(got - ref)
    rn = np.linalg.norm(ref, axis=-1, keepdims=True)
    cos = (got * ref).sum(-1) / (np.linalg.norm(got, axis=-1) * rn[..., 0] + 1e-30)
    return float(err.max()), float((err / (rn + 1e-30)).max()), float(cos.min())


# Accuracy records of this session's parity tests, printed at the end of the
# run (conftest.pytest_terminal_summary).
ACCURACY = []


def accuracy(w: synth.Workload, q, k, v, got, o_int4, b, h, r0, nr):
    """The accuracy record of rows [r0, r0+nr) of head (b, h): max-abs error
    against the oracle's INT4 result, the largest error relative to the row
    norm, and the cosine of the output against unquantised attention (RoPE,
    no rotation, no quantisation, double softmax; oracle.attn_ref)."""
    import oracle
    unq = oracle.attn_ref(q, k, v, w.grid, w.rope_dim, sm_scale(w), b, h, r0, nr, theta=w.theta,
                          phase=w.rope_phase)
    err = np.abs(got - o_int4)
    rn = np.linalg.norm(o_int4, axis=-1)
    cos = (got * unq).sum(-1) / (np.linalg.norm(got, axis=-1) * np.linalg.norm(unq, axis=-1) + 1e-30)
    return {"max_abs_vs_oracle": float(err.max()),
            "max_rel_row_norm": float((err.max(-1) / (rn + 1e-30)).max()),
            "cos_vs_unquantised_mean": float(cos.mean()), "cos_vs_unquantised_min": float(cos.min()),
            "rows": int(nr)}


def report(name: str, rec: dict):
    ACCURACY.append((name, rec))
    return rec
