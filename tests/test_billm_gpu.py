"""The two-plane binary layer of BiLLM's residual approximation
(billm_binarize / billm_linear) against the oracle (BiLLM page, "方法细节：残差
近似与最优断点拆分", step 2).

billm_binarize: the sign planes match the oracle bit for bit and the fp16
scales are the oracle's fp64 scales rounded to fp16 (the two sides sum |W| in
different orders, so the fp64 scales agree to ~1e-15 and the fp16 values may
differ by one unit only at a rounding boundary).
billm_linear: within 2e-3 of the token's largest output against the oracle's
fp64 product (the bar OneBit is held to; the only approximation is the 23-bit
image of x, error <= 2^-23 of the token's max |x| per element), on every
contraction path: the fused streamed kernel (M <= 2), the prepared streamed
kernel (M 3..4) and the tensor-core kernel (M >= 5), at the 7B and 13B layer
shapes, with outlier tokens."""
import numpy as np
import pytest
import torch

from bit_weight_linear_b200 import synth

pytestmark = pytest.mark.gpu

TOL = 2e-3


@pytest.fixture(scope="module")
def blw():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_linear_b200 import build
    build.build()
    import bit_weight_linear_b200 as m
    return m


def _binarize(blw, oref, N, K, seed):
    W = synth.svid_weights(N, K, seed=seed)
    b2, alpha, ao, ar = blw.billm_binarize(W.cuda(), return_alpha64=True)
    torch.cuda.synchronize()
    Bo, Br, ao_ref, ar_ref = oref.billm_binarize(W.numpy())
    return W, b2, alpha, ao, ar, (Bo, Br, ao_ref, ar_ref)


def test_billm_binarize_matches_oracle(blw, oref):
    for (N, K) in [(4096, 4096), (48, 384)]:
        W, b2, alpha, ao, ar, (Bo, Br, ao_ref, ar_ref) = _binarize(blw, oref, N, K, seed=N + K)
        words = b2.cpu().numpy().view(np.uint32)
        assert np.array_equal(words[:N], oref.pack_sign(Bo.astype(np.float16)))
        assert np.array_equal(words[N:], oref.pack_sign(Br.astype(np.float16)))
        assert np.max(np.abs(ao.cpu().numpy() - ao_ref) / ao_ref) <= 1e-13
        assert np.max(np.abs(ar.cpu().numpy() - ar_ref) / ar_ref) <= 1e-13
        a16 = alpha.cpu().numpy()
        ref16 = np.concatenate([ao_ref, ar_ref]).astype(np.float16)
        d = np.abs(a16.view(np.int16).astype(np.int32) - ref16.view(np.int16).astype(np.int32))
        assert d.max() <= 1 and np.mean(d == 0) >= 0.999


def test_billm_binarize_edge_rows(blw, oref):
    """A constant-magnitude row (residual 0: alpha_r = 0, B_r = +1), signed
    zeros, and a non-finite weight (rejected)."""
    N, K = 32, 128
    W = synth.svid_weights(N, K, seed=4)
    W[0] = torch.where(torch.arange(K) % 3 == 0, -0.5, 0.5)
    W[1, :16] = 0.0
    W[1, 16:32] = -0.0
    b2, alpha, ao, ar = blw.billm_binarize(W.cuda(), return_alpha64=True)
    torch.cuda.synchronize()
    Bo, Br, ao_ref, ar_ref = oref.billm_binarize(W.numpy())
    words = b2.cpu().numpy().view(np.uint32)
    assert np.array_equal(words[:N], oref.pack_sign(Bo.astype(np.float16)))
    assert np.array_equal(words[N:], oref.pack_sign(Br.astype(np.float16)))
    assert ao.cpu().numpy()[0] == 0.5 and ar.cpu().numpy()[0] == 0.0
    assert (words[N] == 0xffffffff).all()
    W[2, 3] = float("nan")
    with pytest.raises(blw.BitLinearError, match="INVALID_VALUE"):
        blw.billm_binarize(W.cuda())


@pytest.mark.parametrize("M", [1, 2, 3, 4, 16, 256])
@pytest.mark.parametrize("K,N", [(4096, 4096), (13824, 5120)])
def test_billm_linear_parity(blw, oref, M, K, N):
    W, b2, alpha, *_ = _binarize(blw, oref, N, K, seed=3 * N + K)
    x = synth.activations(M, K, seed=M * 7 + K, outlier_frac=0.01)
    x[0, 17] = 2000.0                          # one dominant activation in token 0
    if M > 1:
        x[M - 1, 5] = -60000.0                 # and a larger one in the last token
    y = blw.billm_linear(x.cuda(), b2, alpha)
    torch.cuda.synchronize()
    words = b2.cpu().numpy().view(np.uint32)
    a = alpha.cpu().numpy()
    _, z_ref = oref.billm_linear(x.numpy(), words[:N], words[N:], a[:N], a[N:], parallel=True)
    yv = y.cpu().numpy().astype(np.float64)
    err = np.max(np.abs(yv - z_ref), axis=1) / np.max(np.abs(z_ref), axis=1)
    assert err.max() <= TOL, err.max()


def test_billm_linear_equals_onebit_sum(blw):
    """The layer is the sum of two OneBit layers with g = 1 and h = alpha_o,
    alpha_r: within the fp16 rounding of the two separate outputs."""
    N, K, M = 1024, 2048, 4
    W = synth.svid_weights(N, K, seed=91)
    b2, alpha = blw.billm_binarize(W.cuda())
    x = synth.activations(M, K, seed=92).cuda()
    y = blw.billm_linear(x, b2, alpha).float()
    ones = torch.ones((K,), dtype=torch.float16, device="cuda")
    yo = blw.ob_linear(x, b2[:N].contiguous(), ones, alpha[:N].contiguous()).float()
    yr = blw.ob_linear(x, b2[N:].contiguous(), ones, alpha[N:].contiguous()).float()
    torch.cuda.synchronize()
    ref = yo + yr
    assert torch.max(torch.abs(y - ref)).item() <= 2.0 ** -9 * torch.max(torch.abs(ref)).item()
