"""ctypes binding of librota_attn.so (include/rota_attn.h), same names.

Argument marshalling only: every step of the attention runs in the CUDA
kernels of the library.  torch is used for device memory and streams.  If the
library is missing the import fails loudly -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "librota_attn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built; run `python -m video_dit_b200.build` "
                      "(or __graft_entry__.build()) first")

_lib = ctypes.CDLL(LIB_PATH)

ROTA_OK, ROTA_ERR_INVALID_ARG, ROTA_ERR_UNSUPPORTED, ROTA_ERR_CUDA, ROTA_ERR_TIMEOUT, ROTA_ERR_DEVICE = range(6)
(ROTA_BUF_Q_CODES, ROTA_BUF_K_CODES, ROTA_BUF_Q_SCALE, ROTA_BUF_K_SCALE, ROTA_BUF_V_CODES,
 ROTA_BUF_V_SCALE, ROTA_BUF_Q_ROPE, ROTA_BUF_K_ROPE, ROTA_BUF_ROPE_TABLE, ROTA_BUF_INT4_WORK,
 ROTA_BUF_COUNT) = range(11)


class rota_attn_desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("grid_t", ctypes.c_int32), ("grid_h", ctypes.c_int32),
                ("grid_w", ctypes.c_int32), ("rope_dim", ctypes.c_int32 * 3),
                ("had_block", ctypes.c_int32 * 3), ("rope_theta", ctypes.c_float),
                ("sm_scale", ctypes.c_float), ("rope_phase", ctypes.c_float * 3),
                ("quant_block", ctypes.c_int32), ("max_group", ctypes.c_int32), ("row_sum", ctypes.c_int32)]


class rota_attn_buffers(ctypes.Structure):
    _fields_ = [("q_codes", ctypes.c_void_p), ("k_codes", ctypes.c_void_p),
                ("q_scale", ctypes.c_void_p), ("k_scale", ctypes.c_void_p),
                ("v_codes", ctypes.c_void_p), ("v_scale", ctypes.c_void_p),
                ("q_rope", ctypes.c_void_p), ("k_rope", ctypes.c_void_p),
                ("rope_cos", ctypes.c_void_p), ("rope_sin", ctypes.c_void_p),
                ("int4_work", ctypes.c_void_p)]


_P = ctypes.c_void_p
_D = ctypes.POINTER(rota_attn_desc)
_BUF = ctypes.POINTER(rota_attn_buffers)
_SIGS = {
    "rota_attn_validate": ([_D], ctypes.c_int),
    "rota_attn_buffer_sizes": ([_D, ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "rota_attn_build_rope_tables": ([_D, _P, _P], ctypes.c_int),
    "rota_attn_prepare_qk": ([_D, _P, _P, _P, _P, _BUF, _P], ctypes.c_int),
    "rota_attn_fwd_int4": ([_D, _BUF, _P, _P, _P], ctypes.c_int),
    "rota_attn_qkv_prepare": ([_D, _P, _P, ctypes.c_int32, _P, _BUF, _P, _P], ctypes.c_int),
    "rota_attn_int4_widen": ([_D, _BUF, _P, _P], ctypes.c_int),
    "rota_attn_int4_attend": ([_D, _BUF, _P, _P, _P], ctypes.c_int),
    "rota_attn_fwd_fp16_fallback": ([_D, _BUF, _P, _P, _P, _P], ctypes.c_int),
    "rota_attn_get_error": ([_P], ctypes.c_int),
    "rota_attn_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "rota_attn_debug_dump_int4": ([_D, _BUF, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                   ctypes.c_int32, _P, _P, _P, _P], ctypes.c_int),
    "rota_attn_debug_pcode": ([_P, _P, ctypes.c_int64, _P], ctypes.c_int),
    "rota_attn_debug_pcode_fma": ([_P, _P, ctypes.c_int64, _P], ctypes.c_int),
    "rota_attn_debug_inject_timeout": ([ctypes.c_int32, ctypes.c_uint64], ctypes.c_int),
    "rota_attn_debug_mma_cycles": ([ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, _P, _P], ctypes.c_int),
    "rota_attn_fwd_int4_noalloc": ([_D, _P, _P, _P, _P, _P], ctypes.c_int),
    "rota_attn_pipeline_create": ([ctypes.c_int32, ctypes.POINTER(_P)], ctypes.c_int),
    "rota_attn_pipeline_destroy": ([_P], ctypes.c_int),
    "rota_attn_pipeline_chunk_heads": ([_D, ctypes.c_int32], ctypes.c_int32),
    "rota_attn_forward_host": ([_D, _P, _P, _P, _P, _P, _P, _P, _P, _P, _BUF, ctypes.c_int32, _P, _P],
                               ctypes.c_int),
    "rota_attn_head_error": ([_D, _P, _P, _P, _P], ctypes.c_int),
    "rota_attn_debug_hadamard": ([ctypes.c_int32, _P], ctypes.c_int),
    "rota_attn_select_fp16_heads": ([_P, ctypes.c_int32, ctypes.c_int32, ctypes.c_float, ctypes.c_int32, _P, _P],
                                    ctypes.c_int),
}
for _name, (_args, _res) in _SIGS.items():
    _f = getattr(_lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class RotaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {rota_attn_status_string(status)} ({status})")
        self.status = status


def _check(status: int, where: str) -> int:
    if status != ROTA_OK:
        raise RotaError(status, where)
    return status


def _ptr(t) -> Optional[int]:
    """Device pointer of a torch tensor (or None)."""
    return None if t is None else int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(getattr(stream, "cuda_stream", stream))


def _flags(head_flags) -> Optional[ctypes.Array]:
    if head_flags is None:
        return None
    f = np.ascontiguousarray(np.asarray(head_flags, dtype=np.uint8))
    return (ctypes.c_uint8 * f.size).from_buffer_copy(f.tobytes())


# ------------------------------------------------------------- raw C ABI ---

def rota_attn_status_string(status: int) -> str:
    return _lib.rota_attn_status_string(int(status)).decode()


def rota_attn_validate(desc: rota_attn_desc) -> int:
    return _lib.rota_attn_validate(ctypes.byref(desc))


def rota_attn_buffer_sizes(desc: rota_attn_desc) -> list:
    out = (ctypes.c_size_t * ROTA_BUF_COUNT)()
    _check(_lib.rota_attn_buffer_sizes(ctypes.byref(desc), out), "rota_attn_buffer_sizes")
    return list(out)


def rota_attn_build_rope_tables(desc: rota_attn_desc):
    n = rota_attn_buffer_sizes(desc)[ROTA_BUF_ROPE_TABLE] // 4
    c = np.empty(n, np.float32)
    s = np.empty(n, np.float32)
    _check(_lib.rota_attn_build_rope_tables(ctypes.byref(desc), c.ctypes.data, s.ctypes.data),
           "rota_attn_build_rope_tables")
    return c, s


def rota_attn_prepare_qk(desc, q, k, v, head_flags, buffers: rota_attn_buffers, stream=None) -> int:
    return _lib.rota_attn_prepare_qk(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _flags(head_flags),
                                     ctypes.byref(buffers), _stream(stream))


def rota_attn_fwd_int4(desc, buffers: rota_attn_buffers, head_flags, out, stream=None) -> int:
    return _lib.rota_attn_fwd_int4(ctypes.byref(desc), ctypes.byref(buffers), _flags(head_flags), _ptr(out),
                                   _stream(stream))


def rota_attn_qkv_prepare(desc, x, w, C: int, head_flags, buffers: rota_attn_buffers, v_out=None,
                          stream=None) -> int:
    return _lib.rota_attn_qkv_prepare(ctypes.byref(desc), _ptr(x), _ptr(w), int(C), _flags(head_flags),
                                      ctypes.byref(buffers), _ptr(v_out), _stream(stream))


def rota_attn_int4_widen(desc, buffers: rota_attn_buffers, head_flags, stream=None) -> int:
    return _lib.rota_attn_int4_widen(ctypes.byref(desc), ctypes.byref(buffers), _flags(head_flags), _stream(stream))


def rota_attn_int4_attend(desc, buffers: rota_attn_buffers, head_flags, out, stream=None) -> int:
    return _lib.rota_attn_int4_attend(ctypes.byref(desc), ctypes.byref(buffers), _flags(head_flags), _ptr(out),
                                      _stream(stream))


def rota_attn_fwd_fp16_fallback(desc, buffers: rota_attn_buffers, v, head_flags, out, stream=None) -> int:
    return _lib.rota_attn_fwd_fp16_fallback(ctypes.byref(desc), ctypes.byref(buffers), _ptr(v),
                                            _flags(head_flags), _ptr(out), _stream(stream))


def rota_attn_fwd_int4_noalloc(desc, q, k, v, out, stream=None) -> int:
    """All-INT4 forward whose intermediates live in the library's static
    device scratch (for callers that cannot allocate device memory)."""
    return _lib.rota_attn_fwd_int4_noalloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(out),
                                           _stream(stream))


def rota_attn_pipeline_create(max_chunks: int):
    """-> (status, handle): copy streams and events on the current device."""
    h = _P()
    st = _lib.rota_attn_pipeline_create(int(max_chunks), ctypes.byref(h))
    return st, h


def rota_attn_pipeline_destroy(handle) -> int:
    return _lib.rota_attn_pipeline_destroy(handle)


def rota_attn_pipeline_chunk_heads(desc, num_sms: int = 0) -> int:
    return _lib.rota_attn_pipeline_chunk_heads(ctypes.byref(desc), int(num_sms))


def rota_attn_forward_host(desc, q_host, k_host, v_host, head_flags, out_host, q_dev, k_dev, v_dev, out_dev,
                           buffers: rota_attn_buffers, heads_per_chunk: int, pipeline, stream=None) -> int:
    return _lib.rota_attn_forward_host(ctypes.byref(desc), _ptr(q_host), _ptr(k_host), _ptr(v_host),
                                       _flags(head_flags), _ptr(out_host), _ptr(q_dev), _ptr(k_dev), _ptr(v_dev),
                                       _ptr(out_dev), ctypes.byref(buffers), int(heads_per_chunk), pipeline,
                                       _stream(stream))


def rota_attn_head_error(desc, out_test, out_ref, sums, stream=None) -> int:
    return _lib.rota_attn_head_error(ctypes.byref(desc), _ptr(out_test), _ptr(out_ref), _ptr(sums),
                                     _stream(stream))


def rota_attn_select_fp16_heads(sums: np.ndarray, B: int, H: int, max_rel_err: float, max_fp16_heads: int = -1):
    """-> (status, flags uint8 [H], rel_err float32 [H]) from host sums [B*H*2]."""
    sums = np.ascontiguousarray(sums, dtype=np.float64)
    flags = np.zeros(H, np.uint8)
    rel = np.zeros(H, np.float32)
    st = _lib.rota_attn_select_fp16_heads(sums.ctypes.data, int(B), int(H), float(max_rel_err),
                                          int(max_fp16_heads), rel.ctypes.data, flags.ctypes.data)
    return st, flags, rel


def rota_attn_get_error(stream=None) -> int:
    return _lib.rota_attn_get_error(_stream(stream))


def rota_attn_debug_dump_int4(desc, buffers, b, h, r0, nr, s_out, p_out, out, stream=None) -> int:
    return _lib.rota_attn_debug_dump_int4(ctypes.byref(desc), ctypes.byref(buffers), b, h, r0, nr,
                                          _ptr(s_out), _ptr(p_out), _ptr(out), _stream(stream))


def rota_attn_debug_pcode(d, u, stream=None) -> int:
    return _lib.rota_attn_debug_pcode(_ptr(d), _ptr(u), int(d.numel()), _stream(stream))


def rota_attn_debug_pcode_fma(d, u, stream=None) -> int:
    return _lib.rota_attn_debug_pcode_fma(_ptr(d), _ptr(u), int(d.numel()), _stream(stream))


def rota_attn_debug_hadamard(n: int):
    """-> (status, int8 [n, n]): the library's Hadamard matrix of a non-power-of-two order."""
    h = np.zeros((max(n, 1), max(n, 1)), np.int8)
    return _lib.rota_attn_debug_hadamard(int(n), h.ctypes.data), h


def rota_attn_debug_mma_cycles(kind: int, n: int, iters: int, cycles, stream=None) -> int:
    return _lib.rota_attn_debug_mma_cycles(int(kind), int(n), int(iters), _ptr(cycles), _stream(stream))


def rota_attn_debug_inject_timeout(arm: bool, timeout_ns: int = 0) -> int:
    return _lib.rota_attn_debug_inject_timeout(int(bool(arm)), int(timeout_ns))


# ---------------------------------------------------- descriptor helpers ---

def default_had_block(d_a: int) -> int:
    b = 1
    while d_a % (2 * b) == 0 and 2 * b <= 64:
        b *= 2
    return b


def make_desc(B: int, H: int, head_dim: int, grid: Sequence[int], rope_dim: Sequence[int],
              had_block: Optional[Sequence[int]] = None, theta: float = 10000.0,
              sm_scale: float = 0.0, rope_phase: Sequence[float] = (0.0, 0.0, 0.0), quant_block: int = 64,
              max_group: int = 64, row_sum: int = 0) -> rota_attn_desc:
    d = rota_attn_desc()
    d.B, d.H, d.head_dim = B, H, head_dim
    d.grid_t, d.grid_h, d.grid_w = grid
    d.N = grid[0] * grid[1] * grid[2]
    d.rope_dim[:] = list(rope_dim)
    d.had_block[:] = list(had_block or [default_had_block(r) for r in rope_dim])
    d.rope_theta = theta
    d.sm_scale = sm_scale
    d.rope_phase[:] = [float(x) for x in rope_phase]
    d.quant_block, d.max_group, d.row_sum = quant_block, max_group, row_sum
    return d


class RotaAttention:
    """Owns the intermediate device buffers of one problem shape (torch
    allocations) and calls the C ABI: prepare -> INT4 attention -> FP16
    fallback for the flagged heads."""

    def __init__(self, desc: rota_attn_desc, device="cuda", need_fp16: bool = True):
        import torch
        _check(rota_attn_validate(desc), "rota_attn_validate")
        self.desc = desc
        self.device = torch.device(device)
        sz = rota_attn_buffer_sizes(desc)

        def u8(n):
            # round up to 16 bytes so every buffer is 16-byte aligned and non-empty
            return torch.empty(max(16, (n + 15) // 16 * 16), dtype=torch.uint8, device=self.device)
        self.q_codes, self.k_codes = u8(sz[ROTA_BUF_Q_CODES]), u8(sz[ROTA_BUF_K_CODES])
        self.q_scale, self.k_scale = u8(sz[ROTA_BUF_Q_SCALE]), u8(sz[ROTA_BUF_K_SCALE])
        self.v_codes, self.v_scale = u8(sz[ROTA_BUF_V_CODES]), u8(sz[ROTA_BUF_V_SCALE])
        self.int4_work = u8(sz[ROTA_BUF_INT4_WORK])
        self.q_rope = u8(sz[ROTA_BUF_Q_ROPE]) if need_fp16 else None
        self.k_rope = u8(sz[ROTA_BUF_K_ROPE]) if need_fp16 else None
        c, s = rota_attn_build_rope_tables(desc)
        self.rope_cos = torch.from_numpy(c).to(self.device)
        self.rope_sin = torch.from_numpy(s).to(self.device)
        b = rota_attn_buffers()
        for name in ("q_codes", "k_codes", "q_scale", "k_scale", "v_codes", "v_scale", "q_rope", "k_rope",
                     "rope_cos", "rope_sin", "int4_work"):
            setattr(b, name, _ptr(getattr(self, name)))
        self.buffers = b

    def prepare(self, q, k, v, head_flags=None, stream=None):
        _check(rota_attn_prepare_qk(self.desc, q, k, v, head_flags, self.buffers, stream), "prepare_qk")

    def attention(self, v, head_flags, out, stream=None):
        _check(rota_attn_fwd_int4(self.desc, self.buffers, head_flags, out, stream), "fwd_int4")
        if head_flags is not None and np.any(np.asarray(head_flags)):
            _check(rota_attn_fwd_fp16_fallback(self.desc, self.buffers, v, head_flags, out, stream),
                   "fwd_fp16_fallback")

    def forward(self, q, k, v, head_flags=None, out=None, stream=None):
        """q, k, v: fp16 [B,H,N,d] device tensors -> fp32 [B,H,N,d]."""
        import torch
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        self.prepare(q, k, v, head_flags, stream)
        self.attention(v, head_flags, out, stream)
        return out

    def forward_host(self, q_host, k_host, v_host, head_flags=None, out_host=None, heads_per_chunk: int = 0,
                     stream=None):
        """q_host, k_host, v_host: fp16 [B,H,N,d] pinned host tensors -> fp32
        [B,H,N,d] host tensor, through rota_attn_forward_host (copies of
        neighbouring head chunks overlap the kernels).  The device staging
        tensors and the copy pipeline are made on first use and kept.  The
        result is complete once `stream` (default: the current stream) has
        reached the end of the call."""
        import torch
        if out_host is None:
            out_host = torch.empty(q_host.shape, dtype=torch.float32, pin_memory=True)
        d = self.desc
        if getattr(self, "_stage", None) is None:
            shape = (d.B, d.H, d.N, d.head_dim)
            self._stage = tuple(torch.empty(shape, dtype=torch.float16, device=self.device) for _ in range(3)) + (
                torch.empty(shape, dtype=torch.float32, device=self.device),)
            st, h = rota_attn_pipeline_create(d.B * d.H)
            _check(st, "rota_attn_pipeline_create")
            self._pipeline = h
        qd, kd, vd, od = self._stage
        _check(rota_attn_forward_host(d, q_host, k_host, v_host, head_flags, out_host, qd, kd, vd, od, self.buffers,
                                      heads_per_chunk, self._pipeline, stream), "rota_attn_forward_host")
        return out_host

    def calibrate_flags(self, q, k, v, max_rel_err: float = 0.1, max_fp16_heads: int = -1, stream=None):
        """Runs the call twice on these inputs -- every head INT4, then every
        head on the FP16 fallback -- and flags the heads whose INT4 output is
        furthest from the FP16 one (rota_attn_head_error +
        rota_attn_select_fp16_heads).  Returns (flags uint8 [H], relative
        error float32 [H]).  Needs the FP16 buffers (need_fp16=True)."""
        import torch
        if self.q_rope is None:
            raise ValueError("calibrate_flags needs a RotaAttention made with need_fp16=True")
        d = self.desc
        shape = (d.B, d.H, d.N, d.head_dim)
        o4 = torch.empty(shape, dtype=torch.float32, device=self.device)
        o16 = torch.empty(shape, dtype=torch.float32, device=self.device)
        self.forward(q, k, v, np.zeros(d.H, np.uint8), o4, stream)
        self.forward(q, k, v, np.ones(d.H, np.uint8), o16, stream)
        sums = torch.empty(d.B * d.H * 2, dtype=torch.float64, device=self.device)
        _check(rota_attn_head_error(d, o4, o16, sums, stream), "rota_attn_head_error")
        _check(rota_attn_get_error(stream), "calibration")
        st, flags, rel = rota_attn_select_fp16_heads(sums.cpu().numpy(), d.B, d.H, max_rel_err, max_fp16_heads)
        _check(st, "rota_attn_select_fp16_heads")
        return flags, rel

    def close(self):
        """Releases the copy pipeline of forward_host (if one was made)."""
        h = getattr(self, "_pipeline", None)
        if h is not None:
            self._pipeline = None
            _check(rota_attn_pipeline_destroy(h), "rota_attn_pipeline_destroy")

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # views of the intermediate buffers in the documented layouts
    def codes(self):
        d = self.desc
        B, H, N, D = d.B, d.H, d.N, d.head_dim
        nblk = (N + 63) // 64
        npad = nblk * 64
        import torch
        f32 = lambda t, n: t[: n * 4].view(torch.float32)
        return dict(
            q_codes=self.q_codes[: B * H * npad * D // 2].view(B, H, npad, D // 2),
            k_codes=self.k_codes[: B * H * npad * D // 2].view(B, H, npad, D // 2),
            q_scale=f32(self.q_scale, B * H * nblk).view(B, H, nblk),
            k_scale=f32(self.k_scale, B * H * nblk).view(B, H, nblk),
            v_codes=self.v_codes[: B * H * nblk * D * 32].view(B, H, nblk, D, 32),
            v_scale=f32(self.v_scale, B * H * nblk * D).view(B, H, nblk, D),
            q_rope=None if self.q_rope is None else self.q_rope[: B * H * N * D * 2].view(torch.int16).view(B, H, N, D),
            k_rope=None if self.k_rope is None else self.k_rope[: B * H * N * D * 2].view(torch.int16).view(B, H, N, D),
        )

