"""Host-side checks of the C ABI: the library loads without a GPU, exports
every function include/rota_attn.h declares, rejects bad arguments before
touching the device, and its host-built RoPE tables equal the oracle's byte
for byte."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
from video_dit_b200 import build as vbuild
from video_dit_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def ra():
    vbuild.build()
    from video_dit_b200 import rota_attn
    return rota_attn


def declared_functions():
    src = open(os.path.join(ROOT, "include", "rota_attn.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rota_attn_\w+)\s*\(", src)))


def test_every_declared_symbol_is_exported(ra):
    names = declared_functions()
    assert len(names) >= 11
    lib = ctypes.CDLL(ra.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def _desc(ra, w):
    return ra.make_desc(w.B, w.H, w.d, w.grid, w.rope_dim, w.had_block, w.theta, rope_phase=w.rope_phase,
                        max_group=w.max_group, row_sum=w.row_sum)


def test_validate_accepts_workloads(ra):
    for w in synth.WORKLOADS.values():
        assert ra.rota_attn_validate(_desc(ra, w)) == ra.ROTA_OK, w.name


@pytest.mark.parametrize("field,value,status", [
    ("N", 1000, 1), ("head_dim", 96, 1), ("B", 0, 1), ("grid_w", 0, 1),
    ("rope_theta", -1.0, 1), ("sm_scale", float("nan"), 1), ("H", 300, 2),
    ("quant_block", 32, 2), ("quant_block", -64, 1), ("max_group", 256, 2), ("max_group", 96, 2),
    ("max_group", -1, 1), ("row_sum", 2, 1), ("row_sum", -1, 1),
])
def test_validate_rejects(ra, field, value, status):
    d = _desc(ra, synth.WORKLOADS["wan480"])
    setattr(d, field, value)
    assert ra.rota_attn_validate(d) == status


@pytest.mark.parametrize("field,value", [("quant_block", 0), ("quant_block", 64), ("max_group", 0), ("max_group", 64),
                                         ("max_group", 128), ("row_sum", 0), ("row_sum", 1)])
def test_validate_accepts_numerics_options(ra, field, value):
    d = _desc(ra, synth.WORKLOADS["wan480"])
    setattr(d, field, value)
    assert ra.rota_attn_validate(d) == ra.ROTA_OK


def test_validate_rejects_bad_partitions(ra):
    d = _desc(ra, synth.WORKLOADS["wan480"])
    d.rope_dim[:] = [43, 43, 42]
    assert ra.rota_attn_validate(d) == ra.ROTA_ERR_INVALID_ARG
    d = _desc(ra, synth.WORKLOADS["wan480"])
    d.had_block[:] = [8, 2, 2]                  # 8 does not divide 44
    assert ra.rota_attn_validate(d) == ra.ROTA_ERR_INVALID_ARG
    d.had_block[:] = [3, 2, 2]
    assert ra.rota_attn_validate(d) == ra.ROTA_ERR_INVALID_ARG
    d = _desc(ra, synth.WORKLOADS["tiny"])
    d.head_dim = 128                             # partitions sum to 64
    assert ra.rota_attn_validate(d) == ra.ROTA_ERR_INVALID_ARG


def test_null_arguments_rejected_on_host(ra):
    d = _desc(ra, synth.WORKLOADS["tiny"])
    b = ra.rota_attn_buffers()
    assert ra._lib.rota_attn_prepare_qk(ctypes.byref(d), None, None, None, None, ctypes.byref(b), None) == 1
    assert ra._lib.rota_attn_fwd_int4(ctypes.byref(d), ctypes.byref(b), None, None, None) == 1
    assert ra._lib.rota_attn_fwd_fp16_fallback(ctypes.byref(d), ctypes.byref(b), None, None, None, None) == 1
    assert ra._lib.rota_attn_debug_pcode(None, None, 5, None) == 1
    assert ra._lib.rota_attn_debug_pcode_fma(None, None, 5, None) == 1
    assert ra._lib.rota_attn_prepare_qk(None, None, None, None, None, None, None) == 1
    assert ra.rota_attn_status_string(4) == "device wait timed out"


def test_buffer_sizes(ra):
    w = synth.WORKLOADS["wan480"]
    sz = ra.rota_attn_buffer_sizes(_desc(ra, w))
    npad = 32768
    assert sz[ra.ROTA_BUF_Q_CODES] == 40 * npad * 64
    assert sz[ra.ROTA_BUF_V_CODES] == 40 * 512 * 128 * 32
    assert sz[ra.ROTA_BUF_V_SCALE] == 40 * 512 * 128 * 4
    assert sz[ra.ROTA_BUF_Q_ROPE] == 40 * 32760 * 128 * 2
    assert sz[ra.ROTA_BUF_ROPE_TABLE] == 4 * (21 * 22 + 30 * 21 + 52 * 21)


@pytest.mark.parametrize("name", ["tiny", "wan480", "wan720", "hunyuan", "wan480_phase"])
def test_rope_tables_identical_to_oracle(ra, name):
    if name == "wan480_phase":   # the merged per-pair rotation: a phase per partition
        w = synth.scaled(synth.WORKLOADS["wan480"], name, rope_phase=(0.3, 0.7853982, -2.5))
    else:
        w = synth.WORKLOADS[name]
    c, s = ra.rota_attn_build_rope_tables(_desc(ra, w))
    oc, os_ = oracle.rope_tables(w.grid, w.rope_dim, w.theta, w.rope_phase)
    assert np.array_equal(c.view(np.uint32), oc.view(np.uint32))
    assert np.array_equal(s.view(np.uint32), os_.view(np.uint32))


# ----------------------------------------------- host-to-host pipeline (host logic)

@pytest.mark.parametrize("name", ["wan480", "wan720", "hunyuan"])
def test_chunk_heads_default_is_one_head_on_large_problems(ra, name):
    # one head's fp16 Q/K/V in and fp32 O out cost more than a chunk's fixed
    # overhead on these sizes, so the unhidden first and last copies decide
    assert ra.rota_attn_pipeline_chunk_heads(_desc(ra, synth.WORKLOADS[name]), 148) == 1


def test_chunk_heads_grows_when_heads_are_small(ra):
    # N = 256: a head is 1 attention CTA, so the per-chunk cost dominates
    w = synth.scaled(synth.WORKLOADS["wan480"], "small", H=40, grid=(1, 4, 64))
    h = ra.rota_attn_pipeline_chunk_heads(_desc(ra, w), 148)
    assert 1 < h <= 40
    # a larger N never asks for more heads per chunk
    prev = h
    for grid in [(1, 16, 64), (1, 64, 64), (4, 64, 64)]:
        cur = ra.rota_attn_pipeline_chunk_heads(_desc(ra, synth.scaled(w, "g", grid=grid)), 148)
        assert 1 <= cur <= prev
        prev = cur


def test_chunk_heads_invalid_descriptor(ra):
    d = _desc(ra, synth.WORKLOADS["wan480"])
    d.head_dim = 96
    assert ra.rota_attn_pipeline_chunk_heads(d, 148) == 0
    # num_sms <= 0 falls back to the B200's 148
    d = _desc(ra, synth.WORKLOADS["wan480"])
    assert ra.rota_attn_pipeline_chunk_heads(d, 0) == ra.rota_attn_pipeline_chunk_heads(d, 148)


def test_pipeline_arguments_rejected_before_any_cuda_call(ra):
    h = ctypes.c_void_p()
    assert ra._lib.rota_attn_pipeline_create(0, ctypes.byref(h)) == ra.ROTA_ERR_INVALID_ARG
    assert ra._lib.rota_attn_pipeline_create(4, None) == ra.ROTA_ERR_INVALID_ARG
    assert ra.rota_attn_pipeline_destroy(None) == ra.ROTA_OK
    d = _desc(ra, synth.WORKLOADS["tiny"])
    b = ra.rota_attn_buffers()
    nul = [None] * 4
    # null host / device pointers and a null pipeline
    assert ra._lib.rota_attn_forward_host(ctypes.byref(d), None, None, None, None, None, *nul, ctypes.byref(b), 0,
                                          None, None) == ra.ROTA_ERR_INVALID_ARG
    d.head_dim = 96
    assert ra._lib.rota_attn_forward_host(ctypes.byref(d), None, None, None, None, None, *nul, ctypes.byref(b), 0,
                                          None, None) == ra.ROTA_ERR_INVALID_ARG


# ----------------------------------------------- FP16-head selection (host rule)

def _sums(rel, ref=1.0):
    """Per-head sums (diff^2, ref^2) giving relative errors `rel` (B rows)."""
    rel = np.atleast_2d(np.asarray(rel, np.float64))
    out = np.zeros(rel.shape + (2,), np.float64)
    out[..., 0] = (rel * ref) ** 2
    out[..., 1] = ref ** 2
    return out.reshape(-1)


def test_select_threshold_and_order(ra):
    st, flags, rel = ra.rota_attn_select_fp16_heads(_sums([0.01, 0.2, 0.05, 0.3, 0.11]), 1, 5, 0.1)
    assert st == ra.ROTA_OK
    assert flags.tolist() == [0, 1, 0, 1, 1]
    assert np.allclose(rel, [0.01, 0.2, 0.05, 0.3, 0.11], rtol=1e-6)
    # a budget keeps the worst ones
    _, flags, _ = ra.rota_attn_select_fp16_heads(_sums([0.01, 0.2, 0.05, 0.3, 0.11]), 1, 5, 0.1, 2)
    assert flags.tolist() == [0, 1, 0, 1, 0]
    _, flags, _ = ra.rota_attn_select_fp16_heads(_sums([0.01, 0.2, 0.05, 0.3, 0.11]), 1, 5, 0.1, 0)
    assert not flags.any()
    # nothing above the threshold
    _, flags, _ = ra.rota_attn_select_fp16_heads(_sums([0.01, 0.02]), 1, 2, 0.5)
    assert not flags.any()


def test_select_worst_batch_entry_and_ties(ra):
    # B = 2: head 0 is fine in entry 0 but bad in entry 1
    s = _sums([[0.01, 0.2, 0.2], [0.4, 0.01, 0.2]])
    _, flags, rel = ra.rota_attn_select_fp16_heads(s, 2, 3, 0.1, 2)
    assert np.allclose(rel, [0.4, 0.2, 0.2], rtol=1e-6)
    assert flags.tolist() == [1, 1, 0]            # tie between heads 1 and 2: the lower index


def test_select_degenerate_sums(ra):
    s = _sums([0.0, 0.0, 0.0, 0.0])
    s[2 * 1] = np.nan                             # NaN difference: infinite error
    s[2 * 2 + 1] = 0.0                            # zero reference, zero difference: error 0
    s[2 * 3], s[2 * 3 + 1] = 1.0, 0.0             # zero reference, non-zero difference: infinite
    _, flags, rel = ra.rota_attn_select_fp16_heads(s, 1, 4, 0.1)
    assert flags.tolist() == [0, 1, 0, 1]
    assert np.isinf(rel[1]) and np.isinf(rel[3]) and rel[2] == 0.0


@pytest.mark.parametrize("B,H,thr", [(0, 4, 0.1), (1, 0, 0.1), (1, 257, 0.1), (1, 4, -1.0), (1, 4, float("nan"))])
def test_select_rejects(ra, B, H, thr):
    s = np.zeros(max(1, B) * max(1, H) * 2)
    flags = np.zeros(max(1, H), np.uint8)
    st = ra._lib.rota_attn_select_fp16_heads(s.ctypes.data, B, H, thr, -1, None, flags.ctypes.data)
    assert st == ra.ROTA_ERR_INVALID_ARG


def test_select_rejects_null_pointers(ra):
    s = np.zeros(8)
    flags = np.zeros(4, np.uint8)
    assert ra._lib.rota_attn_select_fp16_heads(None, 1, 4, 0.1, -1, None, flags.ctypes.data) == ra.ROTA_ERR_INVALID_ARG
    assert ra._lib.rota_attn_select_fp16_heads(s.ctypes.data, 1, 4, 0.1, -1, None, None) == ra.ROTA_ERR_INVALID_ARG


def test_validate_rejects_non_finite_phase(ra):
    d = _desc(ra, synth.WORKLOADS["wan480"])
    d.rope_phase[1] = float("inf")
    assert ra.rota_attn_validate(d) == ra.ROTA_ERR_INVALID_ARG
    d.rope_phase[1] = float("nan")
    assert ra.rota_attn_validate(d) == ra.ROTA_ERR_INVALID_ARG
    d.rope_phase[1] = -3.0
    assert ra.rota_attn_validate(d) == ra.ROTA_OK


@pytest.mark.parametrize("had,ok", [((44, 2, 2), True), ((4, 42, 42), False), ((12, 2, 2), False),
                                    ((44, 6, 2), False), ((4, 14, 14), False)])
def test_validate_hadamard_orders(ra, had, ok):
    # 44 = Paley I (q = 43); 42 and 14 (which divide 42) and 6 are orders with no
    # Hadamard matrix; 12 is one but does not divide 44
    d = _desc(ra, synth.scaled(synth.WORKLOADS["wan480"], "v", had=had))
    assert ra.rota_attn_validate(d) == (ra.ROTA_OK if ok else ra.ROTA_ERR_INVALID_ARG)


@pytest.mark.parametrize("had", [(16, 56, 56), (16, 28, 28), (16, 8, 8)])
def test_validate_hunyuan_orders(ra, had):
    d = _desc(ra, synth.scaled(synth.WORKLOADS["hunyuan"], "v", had=had))
    assert ra.rota_attn_validate(d) == ra.ROTA_OK


@pytest.mark.parametrize("n", range(2, 65))
def test_library_hadamard_equals_oracle(ra, n):
    """The library builds its non-power-of-two Hadamard matrices independently
    of the oracle; bit-exact codes need the very same matrix for every order."""
    st, h = ra.rota_attn_debug_hadamard(n)
    ref = oracle.hadamard(n)
    if ref is None:
        assert st == ra.ROTA_ERR_UNSUPPORTED, n
    else:
        assert st == ra.ROTA_OK, n
        assert np.array_equal(h, ref), n


@pytest.mark.parametrize("kind,n,iters,ptr", [(3, 128, 8, 64), (-1, 128, 8, 64), (0, 96, 8, 64), (1, 128, 0, 64),
                                               (2, 256, 65537, 64), (0, 64, 8, 0), (0, 64, 8, 4)])
def test_mma_cycles_rejects_arguments_on_host(ra, kind, n, iters, ptr):
    """Invalid kind, shape, iteration count or output pointer: refused before
    any CUDA call (the pointers are never dereferenced)."""
    assert ra._lib.rota_attn_debug_mma_cycles(kind, n, iters, ptr or None, None) == ra.ROTA_ERR_INVALID_ARG
