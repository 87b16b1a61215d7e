"""The host-to-host forward (head chunks with the copies of neighbouring
chunks overlapping the kernels) returns exactly what the device-resident
calls return on the whole problem, for several chunk sizes, with FP16
fallback heads mixed in, B > 1 and a ragged last chunk; and it refuses a
pipeline with too few events without enqueueing anything."""
import numpy as np
import pytest

from video_dit_b200 import synth

from gpu_util import desc_of, lib, to_dev

pytestmark = pytest.mark.gpu

W = synth.scaled(synth.WORKLOADS["wan480"], "fh", H=5, grid=(2, 7, 11))        # N=154, ragged tail


def _pinned(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


@pytest.mark.parametrize("w,hpc,flags", [
    (W, 0, None), (W, 1, None), (W, 2, [0, 1, 0, 0, 1]), (W, 5, [1, 0, 0, 0, 0]), (W, 3, [0, 0, 1, 1, 0]),
])
def test_forward_host_equals_device_forward(w, hpc, flags):
    import torch
    ra = lib()
    q, k, v = synth.make_inputs(w, seed=3)
    fl = None if flags is None else np.asarray(flags, np.uint8)
    ref_att = ra.RotaAttention(desc_of(w), need_fp16=True)
    ref = ref_att.forward(to_dev(q), to_dev(k), to_dev(v), fl).cpu().numpy()

    att = ra.RotaAttention(desc_of(w), need_fp16=True)
    out_h = torch.full(q.shape, float("nan"), dtype=torch.float32).pin_memory()
    qh, kh, vh = _pinned(q), _pinned(k), _pinned(v)      # alive until the copies are done
    att.forward_host(qh, kh, vh, fl, out_h, heads_per_chunk=hpc)
    st = ra.rota_attn_get_error()
    assert st == ra.ROTA_OK, ra.rota_attn_status_string(st)
    assert np.array_equal(out_h.numpy(), ref)
    att.close()


def test_forward_host_batch_of_two():
    ra = lib()
    w = synth.scaled(W, "fh_b2", H=3, B=2)
    q, k, v = synth.make_inputs(w, seed=4)
    ref = ra.RotaAttention(desc_of(w), need_fp16=False).forward(to_dev(q), to_dev(k), to_dev(v)).cpu().numpy()
    att = ra.RotaAttention(desc_of(w), need_fp16=False)
    qh, kh, vh = _pinned(q), _pinned(k), _pinned(v)
    out_h = att.forward_host(qh, kh, vh, None, heads_per_chunk=2)
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    assert np.array_equal(out_h.numpy(), ref)
    att.close()


def test_forward_host_too_few_events():
    import torch
    ra = lib()
    w = W
    q, k, v = synth.make_inputs(w, seed=3)
    att = ra.RotaAttention(desc_of(w), need_fp16=False)
    st, pl = ra.rota_attn_pipeline_create(2)           # room for 2 chunks; 5 are needed at 1 head each
    assert st == ra.ROTA_OK
    dev = [torch.empty(q.shape, dtype=t, device="cuda") for t in (torch.float16,) * 3 + (torch.float32,)]
    out_h = torch.zeros(q.shape, dtype=torch.float32).pin_memory()
    qh, kh, vh = _pinned(q), _pinned(k), _pinned(v)
    st = ra.rota_attn_forward_host(att.desc, qh, kh, vh, None, out_h, *dev, att.buffers, 1, pl)
    assert st == ra.ROTA_ERR_UNSUPPORTED
    assert ra.rota_attn_pipeline_destroy(pl) == ra.ROTA_OK
    assert ra.rota_attn_get_error() == ra.ROTA_OK


def test_fp16_rows_past_n_do_not_depend_on_neighbouring_memory():
    """An FP16 head followed by an INT4 head: the fallback's Q view runs past the
    head's N into the next head's RoPE rows, which no call writes.  Filled with
    different byte patterns beforehand (0, large fp16 values, moderate ones),
    the outputs must agree bit for bit."""
    ra = lib()
    w = W
    q, k, v = synth.make_inputs(w, seed=3)
    fl = np.asarray([0, 0, 0, 1, 0], np.uint8)
    att = ra.RotaAttention(desc_of(w), need_fp16=True)
    qd, kd, vd = to_dev(q), to_dev(k), to_dev(v)
    outs = []
    for pattern in (0x00, 0x7B, 0x5A):
        att.q_rope.fill_(pattern)
        att.k_rope.fill_(pattern)
        outs.append(att.forward(qd, kd, vd, fl).cpu().numpy())
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    assert np.array_equal(outs[0], outs[1]) and np.array_equal(outs[0], outs[2])
