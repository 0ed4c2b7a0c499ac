"""The bounded device-side waits, made to run out on purpose (never by a GPU
fault): bl_debug_stall_next_launch leaves the first pipeline stage of CTA 0 of
the next launch unrequested, a flag nothing will set.  The kernel's wait gives
up after the short limit, records BL_ERR_TIMEOUT, lets the copies it did issue
land, frees its tensor memory and returns; bl_device_status reports the
timeout once, and the next ordinary call on the same stream is exact again."""
import numpy as np
import pytest
import torch

from bit_weight_linear_b200 import synth

pytestmark = pytest.mark.gpu

LIMIT_NS = 10_000_000   # 10 ms


@pytest.fixture(scope="module")
def blw():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_linear_b200 import build
    build.build()
    import bit_weight_linear_b200 as m
    return m


# M = 1: the streamed decode kernel; M = 32: the whole-tile tensor-core kernel
@pytest.mark.parametrize("M,K,N", [(1, 4096, 1024), (32, 1024, 256)])
def test_stalled_wait_reports_timeout_and_the_next_call_is_exact(blw, oref, M, K, N):
    x = synth.activations(M, K, seed=5_000 + M)
    w = synth.ternary_weights(N, K, seed=5_001 + M)
    w2 = blw.bl_pack_ternary(w.cuda())
    xd = x.cuda()
    assert blw.bl_device_status() == 0
    L = blw.lib()
    assert L.bl_debug_stall_next_launch(LIMIT_NS) == 0
    blw.bl_ternary_linear(xd, w2, 0.02)
    assert blw.bl_device_status() == 6          # BL_ERR_TIMEOUT, reported once
    assert blw.bl_device_status() == 0
    y, acc = blw.bl_ternary_linear(xd, w2, 0.02, return_acc=True)
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), oref.pack_ternary(w.numpy()), 0.02)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert np.array_equal(y.cpu().numpy().view(np.uint16), y_ref.view(np.uint16))


def test_cancelled_stall_changes_nothing(blw):
    L = blw.lib()
    assert L.bl_debug_stall_next_launch(LIMIT_NS) == 0
    assert L.bl_debug_stall_next_launch(0) == 0
    x = synth.activations(1, 1024, seed=5_100).cuda()
    w2 = blw.bl_pack_ternary(synth.ternary_weights(256, 1024, seed=5_101).cuda())
    blw.bl_ternary_linear(x, w2, 0.02)
    assert blw.bl_device_status() == 0
