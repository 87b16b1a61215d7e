"""CPU oracle for RotateAttention's INT4 attention forward (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``video_dit_b200``) never imports it, and the two share no
code: this wrapper only marshals numpy arrays into ``rota_oracle.c``.

Every function cites, in ``rota_oracle.c``, the step of "RotateAttention:
RoPE-Aware Rotation and Range Rectification for INT4 Quantized Attention in
Video Generation" (abstract, Key Points) it states, with the reading taken
where the page is silent.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rota_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fno-unsafe-math-optimizations"]


def build(force: bool = False) -> str:
    """Compile rota_oracle.c into liboracle.so with gcc (plain C, libm only)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32, f32, f64, i64 = ctypes.c_int, ctypes.c_float, ctypes.c_double, ctypes.c_long
        L.oracle_half_to_float.argtypes = [ctypes.c_uint16]
        L.oracle_half_to_float.restype = f32
        L.oracle_float_to_half.argtypes = [f32]
        L.oracle_float_to_half.restype = ctypes.c_uint16
        L.oracle_rope_table_len.argtypes = [P, P]
        L.oracle_rope_table_len.restype = i64
        L.oracle_rope_tables.argtypes = [P, P, f64, P, P, P]
        L.oracle_rope_tables.restype = None
        L.oracle_rope_rotate_row.argtypes = [P, P, i64, P, P, P, P, P, i32, i32]
        L.oracle_rope_rotate_row.restype = None
        L.oracle_quant_params.argtypes = [f32, P, P]
        L.oracle_quant_params.restype = None
        L.oracle_quant_code.argtypes = [f32, f32]
        L.oracle_quant_code.restype = i32
        L.oracle_pack_codes.argtypes = [P, i64, P]
        L.oracle_pack_codes.restype = None
        L.oracle_code_at.argtypes = [P, i64]
        L.oracle_code_at.restype = i32
        L.oracle_quant_codes.argtypes = [P, i64, f32, P]
        L.oracle_quant_codes.restype = None
        L.oracle_prepare.argtypes = [i32, i32, i32, i32, P, P, P, f64, P] + [P] * 12
        L.oracle_prepare.restype = i32
        L.oracle_pcode.argtypes = [f32, P]
        L.oracle_pcode.restype = i32
        L.oracle_pcode_array.argtypes = [P, P, i64, P]
        L.oracle_pcode_array.restype = None
        L.oracle_qkv_project.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P]
        L.oracle_qkv_project.restype = None
        L.oracle_attn_int4.argtypes = [i32, i32, i32, i32, f32, i32, i32] + [P] * 6 + \
            [i32, i32, i32, i32, i32, P, P, P]
        L.oracle_attn_int4.restype = i32
        L.oracle_attn_fp16.argtypes = [i32, i32, i32, i32, f32, P, P, P, i32, i32, i32, i32, P]
        L.oracle_attn_fp16.restype = i32
        L.oracle_attn_ref.argtypes = [i32, i32, i32, i32, P, P, f64, P, f32, P, P, P,
                                      i32, i32, i32, i32, P]
        L.oracle_attn_ref.restype = i32
        L.oracle_hadamard.argtypes = [i32, P]
        L.oracle_hadamard.restype = i32
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _i3(v) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(v, dtype=np.int32).reshape(3))


def _h(a) -> np.ndarray:
    """fp16 array (or its uint16 bits) -> contiguous uint16 bits."""
    a = np.asarray(a)
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16
    return np.ascontiguousarray(a)


# ---------------------------------------------------------------- scalars ---

def half_to_float(bits: int) -> float:
    return float(lib().oracle_half_to_float(int(bits)))


def float_to_half(x: float) -> int:
    return int(lib().oracle_float_to_half(float(x)))


def pcode(d: float) -> int:
    bad = ctypes.c_int(0)
    u = lib().oracle_pcode(float(d), ctypes.byref(bad))
    if bad.value:
        raise ArithmeticError(f"P code of {d!r} is within the tie margin")
    return int(u)


def pcode_array(d: np.ndarray) -> np.ndarray:
    d = np.ascontiguousarray(d, dtype=np.float32)
    u = np.empty(d.shape, np.uint8)
    bad = ctypes.c_int(0)
    lib().oracle_pcode_array(_p(d), _p(u), d.size, ctypes.byref(bad))
    if bad.value:
        raise ArithmeticError("a P code fell within the tie margin")
    return u


def quant_params(amax: float):
    s, i = ctypes.c_float(), ctypes.c_float()
    lib().oracle_quant_params(float(amax), ctypes.byref(s), ctypes.byref(i))
    return s.value, i.value


def quant_code(y: float, inv: float) -> int:
    return int(lib().oracle_quant_code(float(y), float(inv)))


def quant_codes(y: np.ndarray, inv: float) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32)
    c = np.empty(y.shape, np.int8)
    lib().oracle_quant_codes(_p(y), y.size, float(inv), _p(c))
    return c


# ------------------------------------------------------------------- RoPE ---

def _phase(phase) -> np.ndarray:
    """Per-partition RoPE phase as the library stores it (fp32), widened to double."""
    return np.ascontiguousarray(np.asarray(phase, np.float32).astype(np.float64).reshape(3))


def rope_tables(grid, rope_dim, theta: float = 10000.0, phase=(0.0, 0.0, 0.0)):
    g, r = _i3(grid), _i3(rope_dim)
    n = lib().oracle_rope_table_len(_p(g), _p(r))
    c = np.empty(n, np.float32)
    s = np.empty(n, np.float32)
    ph = _phase(phase)
    lib().oracle_rope_tables(_p(g), _p(r), float(theta), _p(ph), _p(c), _p(s))
    return c, s


def hadamard(n: int):
    """The oracle's Hadamard matrix of a non-power-of-two order n (int8 +1/-1,
    n x n), or None if it builds none of that order."""
    h = np.zeros((n, n), np.int8) if n > 0 else np.zeros((1, 1), np.int8)
    ok = lib().oracle_hadamard(int(n), _p(h))
    return h if ok else None


def rope_rotate_row(x: np.ndarray, n: int, grid, rope_dim, had_block, theta: float = 10000.0,
                    rope: bool = True, rotate: bool = True, phase=(0.0, 0.0, 0.0)) -> np.ndarray:
    """RoPE (token index n) then the block Hadamard rotation on one fp32 row."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.empty_like(x)
    c, s = rope_tables(grid, rope_dim, theta, phase)
    g, r, hb = _i3(grid), _i3(rope_dim), _i3(had_block)
    lib().oracle_rope_rotate_row(_p(x), _p(y), int(n), _p(g), _p(r), _p(hb), _p(c), _p(s),
                                 int(rope), int(rotate))
    return y


# --------------------------------------------------------------- pipeline ---

def prepare(q, k, v, grid, rope_dim, had_block, theta=10000.0, flags=None, phase=(0.0, 0.0, 0.0)):
    """The prologue: returns a dict of the library-layout buffers.

    q, k, v: fp16 [B,H,N,d].  flags: uint8 [H] (1 = FP16 fallback head).
    phase: per-partition RoPE phase (the merged rotation; 0 = plain RoPE).
    """
    q, k, v = _h(q), _h(k), _h(v)
    B, H, N, d = q.shape
    nblk = (N + 63) // 64
    npad = nblk * 64
    flags = np.zeros(H, np.uint8) if flags is None else np.ascontiguousarray(flags, np.uint8)
    out = dict(
        q_codes=np.zeros((B, H, npad, d // 2), np.uint8),
        k_codes=np.zeros((B, H, npad, d // 2), np.uint8),
        q_scale=np.zeros((B, H, nblk), np.float32),
        k_scale=np.zeros((B, H, nblk), np.float32),
        v_codes=np.zeros((B, H, nblk, d, 32), np.uint8),
        v_scale=np.zeros((B, H, nblk, d), np.float32),
        q_rope=np.zeros((B, H, N, d), np.uint16),
        k_rope=np.zeros((B, H, N, d), np.uint16),
    )
    g, r, hb = _i3(grid), _i3(rope_dim), _i3(had_block)
    ph = _phase(phase)
    rc = lib().oracle_prepare(B, H, N, d, _p(g), _p(r), _p(hb), float(theta), _p(ph),
                              _p(q), _p(k), _p(v), _p(flags),
                              _p(out["q_codes"]), _p(out["k_codes"]), _p(out["q_scale"]),
                              _p(out["k_scale"]), _p(out["v_codes"]), _p(out["v_scale"]),
                              _p(out["q_rope"]), _p(out["k_rope"]))
    if rc != 0:
        raise MemoryError("oracle_prepare failed")
    return out


def qkv_project(x, w, H: int, D: int):
    """The QKV projection in front of the path: x fp16 [B, N, C], w fp16
    [3 H D, C] -> fp16 q, k, v [B, H, N, D] (exact sums, rounded to fp32 and
    then to fp16)."""
    x, w = _h(x), _h(w)
    B, N, C = x.shape
    q = np.zeros((B, H, N, D), np.uint16)
    k = np.zeros_like(q)
    v = np.zeros_like(q)
    lib().oracle_qkv_project(B, N, C, H, D, _p(x), _p(w), _p(q), _p(k), _p(v))
    return q.view(np.float16), k.view(np.float16), v.view(np.float16)


def attn_int4(prep: dict, N: int, sm_scale: float, b: int, h: int, r0: int, nr: int,
              group: int = 64, online: bool = False, dump: bool = False, rowsum: int = 0):
    """INT4 attention rows [r0, r0+nr) of head (b,h).  Returns out [nr,d] (double)
    and, if dump, S_int [nr,N] int32 and P codes [nr,N] uint8.  group: key group
    of the running max (64 or 128); rowsum: 0 = sum of the codes (R2), 1 = sum
    of the unquantised 15 * 2^d (R1)."""
    qc = prep["q_codes"]
    B, H, _, dh = qc.shape
    d = dh * 2
    out = np.zeros((nr, d), np.float64)
    s = np.zeros((nr, N), np.int32) if dump else None
    p = np.zeros((nr, N), np.uint8) if dump else None
    bad = lib().oracle_attn_int4(B, H, N, d, float(sm_scale), int(group), int(rowsum),
                                 _p(qc), _p(prep["k_codes"]), _p(prep["q_scale"]),
                                 _p(prep["k_scale"]), _p(prep["v_codes"]), _p(prep["v_scale"]),
                                 b, h, r0, nr, int(online),
                                 _p(s) if dump else None, _p(p) if dump else None, _p(out))
    if bad != 0:
        raise ArithmeticError(f"oracle_attn_int4: {bad} range/margin violations")
    return (out, s, p) if dump else out


def attn_fp16(q_rope, k_rope, v, sm_scale: float, b: int, h: int, r0: int, nr: int):
    q_rope, k_rope, v = _h(q_rope), _h(k_rope), _h(v)
    B, H, N, d = q_rope.shape
    out = np.zeros((nr, d), np.float64)
    lib().oracle_attn_fp16(B, H, N, d, float(sm_scale), _p(q_rope), _p(k_rope), _p(v),
                           b, h, r0, nr, _p(out))
    return out


def attn_ref(q, k, v, grid, rope_dim, sm_scale: float, b: int, h: int, r0: int, nr: int,
             theta: float = 10000.0, phase=(0.0, 0.0, 0.0)):
    """Unquantised attention (RoPE, no rotation, double softmax) for the report."""
    q, k, v = _h(q), _h(k), _h(v)
    B, H, N, d = q.shape
    out = np.zeros((nr, d), np.float64)
    g, r = _i3(grid), _i3(rope_dim)
    ph = _phase(phase)
    lib().oracle_attn_ref(B, H, N, d, _p(g), _p(r), float(theta), _p(ph), float(sm_scale),
                          _p(q), _p(k), _p(v), b, h, r0, nr, _p(out))
    return out


def pack_codes(v: np.ndarray) -> np.ndarray:
    """Codes in [-7, 7] (last axis a multiple of 8) -> the packed byte layout."""
    v = np.ascontiguousarray(v, dtype=np.int32)
    out = np.empty(v.shape[:-1] + (v.shape[-1] // 2,), np.uint8)
    lib().oracle_pack_codes(_p(v), v.size, _p(out))
    return out


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """Packed code bytes -> int8 codes (last axis doubled), via the oracle's reader."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    n = packed.shape[-1] * 2
    flat = packed.reshape(-1, packed.shape[-1])
    out = np.empty((flat.shape[0], n), np.int8)
    L = lib()
    for r in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[r])
        out[r] = [L.oracle_code_at(_p(row), i) for i in range(n)]
    return out.reshape(packed.shape[:-1] + (n,))
