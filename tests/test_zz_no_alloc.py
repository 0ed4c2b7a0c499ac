"""bl_ternary_linear_noalloc: the BitLinear forward for callers that cannot
allocate device memory where they run the layer (for example a plugin whose
host program owns all device memory and hands it no allocator, or a loop whose
rules forbid cudaMalloc because it can block the whole device).  It uses the
library's fixed scratch array instead of a caller workspace.

Its results must equal bl_ternary_linear's (the same kernels) and the oracle's
(int32 accumulators and fp16 outputs bit for bit), on calls in a row that reuse
the shared array.

This file is collected last on purpose: it runs after every other test, and it
also passes alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from bit_weight_linear_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blw():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_linear_b200 import build
    build.build()
    import bit_weight_linear_b200 as m
    return m


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# In order: the tensor-core path (M = 96), its small-token tiles (M = 12), the
# activation kernel + prepared streamed kernel (M = 4 on 13824-long rows), and
# the single-kernel streamed path (M = 1); each later call reads a region of
# the shared array an earlier call left behind.
CALLS = [(96, 2048, 512, 1), (12, 4096, 1024, 2), (4, 13824, 256, 3), (1, 4096, 4096, 4)]


def test_noalloc_matches_oracle_and_workspace_entry_point_on_calls_in_a_row(blw, oref):
    L = blw.lib()
    stream = torch.cuda.current_stream().cuda_stream
    for M, K, N, seed in CALLS:
        x = synth.activations(M, K, seed=seed, outlier_frac=0.01)
        w = synth.ternary_weights(N, K, seed=seed + 10)
        w2 = blw.bl_pack_ternary(w.cuda())
        xd = x.cuda()
        y_ws, acc_ws = blw.bl_ternary_linear(xd, w2, 0.02, return_acc=True)
        y = torch.empty((M, N), dtype=torch.float16, device="cuda")
        acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
        st = L.bl_ternary_linear_noalloc(_p(xd), M, K, N, _p(w2), 0.02, _p(y), _p(acc), stream)
        assert st == 0, L.bl_status_string(st)
        torch.cuda.synchronize()
        assert blw.bl_device_status() == 0
        y_ref, acc_ref = oref.ternary_linear(x.numpy(), oref.pack_ternary(w.numpy()), 0.02)
        assert np.array_equal(acc.cpu().numpy(), acc_ref), (M, K, N)
        assert np.array_equal(y.cpu().numpy().view(np.uint16), y_ref.view(np.uint16)), (M, K, N)
        assert torch.equal(acc, acc_ws)
        assert torch.equal(y.view(torch.int16), y_ws.view(torch.int16))


def test_noalloc_rejects_shapes_beyond_its_scratch(blw):
    L = blw.lib()
    x = torch.zeros((1, 128), dtype=torch.float16, device="cuda")
    # M*K = 4096 * 4096 int8 activations plus the per-token scalars exceed 16 MiB;
    # the check happens before any pointer is touched
    st = L.bl_ternary_linear_noalloc(_p(x), 4096, 4096, 16, _p(x), 1.0, _p(x), None, None)
    assert st == 8
    assert L.bl_status_string(8).startswith(b"BL_ERR_SCRATCH_LIMIT")
