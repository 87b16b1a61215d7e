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
    return lib().make_desc(w.B, w.H, w.d, w.grid, w.rope_dim, w.had_block, w.theta, rope_phase=w.rope_phase)


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


def sm_scale(w):
    return float(np.float32(1 / math.sqrt(w.d)))


def row_stats(got, ref):
    """max-abs error, max error relative to the row norm, min cosine."""
    err = np.abs(got - ref)
    rn = np.linalg.norm(ref, axis=-1, keepdims=True)
    cos = (got * ref).sum(-1) / (np.linalg.norm(got, axis=-1) * rn[..., 0] + 1e-30)
    return float(err.max()), float((err / (rn + 1e-30)).max()), float(cos.min())
