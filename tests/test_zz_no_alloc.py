"""bl_ternary_linear_noalloc: the BitLinear forward for callers that cannot
allocate device memory (e.g. a plugin whose host program owns all device memory,
or a loop where allocation is forbidden).  It uses the library's fixed scratch
array instead of a caller workspace, and must give what bl_ternary_linear gives.

This file is collected last on purpose: it runs after every other test, and also
passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from bit_weight_linear_b200 import synth

pytestmark = pytest.mark.gpu

BL_TOL = 1e-3


@pytest.fixture(scope="module")
def blw():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_linear_b200 import build
    build.build()
    import bit_weight_linear_b200 as m
    return m


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row(blw):
    L = blw.lib()
    stream = torch.cuda.current_stream().cuda_stream
    # first a prefill-sized call (tensor-core path), then a decode-sized one that
    # reads a smaller region of the same scratch array the first call left behind
    for M, K, N, seed in [(96, 2048, 512, 1), (4, 4096, 4096, 2)]:
        x = synth.activations(M, K, seed=seed).cuda()
        w2 = blw.bl_pack_ternary(synth.ternary_weights(N, K, seed=seed + 10).cuda())
        y_ref, acc_ref = blw.bl_ternary_linear(x, w2, 0.02, return_acc=True)
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        st = L.bl_ternary_linear_noalloc(_p(x), M, K, N, _p(w2), 0.02, _p(y), _p(acc), stream)
        assert st == 0, L.bl_status_string(st)
        torch.cuda.synchronize()
        assert torch.equal(acc, acc_ref)
        yd = y.float().cpu().numpy().astype(np.float64)
        yr = y_ref.float().cpu().numpy().astype(np.float64)
        assert np.max(np.abs(yd - yr)) <= BL_TOL * np.max(np.abs(yr))


def test_noalloc_rejects_shapes_beyond_its_scratch(blw):
    L = blw.lib()
    x = torch.zeros((1, 128), dtype=torch.float16, device="cuda")
    # M*K = 4096 * 4096 int8 activations plus the per-token scalars exceed 16 MiB;
    # the check happens before any pointer is touched
    st = L.bl_ternary_linear_noalloc(_p(x), 4096, 4096, 16, _p(x), 1.0, _p(x), None, None)
    assert st == 8
    assert L.bl_status_string(8).startswith(b"BL_ERR_SCRATCH_LIMIT")
