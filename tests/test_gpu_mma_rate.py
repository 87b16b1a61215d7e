"""The tcgen05 MMA-rate measurement (rota_attn_debug_mma_cycles) on the device:
every kind and shape completes, and the cycles per MMA are in the range one
MMA of that size can take (at least the issue of one instruction, at most a
dependent chain of full-latency MMAs)."""
import pytest

from gpu_util import lib

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind", [0, 1, 2])
@pytest.mark.parametrize("n", [64, 128, 256])
def test_mma_cycles_every_kind_and_shape(kind, n):
    import torch
    ra = lib()
    cyc = torch.zeros(1, dtype=torch.int64, device="cuda")
    iters = 256
    assert ra.rota_attn_debug_mma_cycles(kind, n, iters, cyc) == ra.ROTA_OK
    torch.cuda.synchronize()
    assert ra.rota_attn_get_error() == ra.ROTA_OK
    per = int(cyc.item()) / (4 * iters)
    assert 8 <= per <= 2000, per
