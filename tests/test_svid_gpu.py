"""SVID initialisation on the device (ob_svid) against the oracle's power
iteration (OneBit page, "2. 基于 SVID 初始化量化模型").

Both sides run the same iteration in fp64 from the same start; they differ
only in summation order, so sigma, a and b agree to ~1e-12 relative and the
tests hold them to 1e-9.  The signs are bit-exact; g = fp16(b) and h = fp16(a)
are equal except where b (a) lies within that 1e-9 of an fp16 rounding
boundary, where they may differ by one unit in the last place."""
import numpy as np
import pytest
import torch

from bit_weight_linear_b200 import synth

pytestmark = pytest.mark.gpu

REL = 1e-9


@pytest.fixture(scope="module")
def blw():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_linear_b200 import build
    build.build()
    import bit_weight_linear_b200 as m
    return m


def _ulp_close(x16: np.ndarray, ref64: np.ndarray):
    ref16 = ref64.astype(np.float16)
    xb, rb = x16.view(np.int16).astype(np.int32), ref16.view(np.int16).astype(np.int32)
    assert np.max(np.abs(xb - rb)) <= 1
    assert np.mean(xb == rb) >= 0.999


def _check(blw, oref, W, max_iter=1000, tol=1e-12):
    s1, g, h, sigma, iters, a, b = blw.ob_svid(W.cuda(), max_iter=max_iter, tol=tol, return_ab=True)
    torch.cuda.synchronize()
    S, a_ref, b_ref, sig_ref, it_ref = oref.svid(W.numpy(), max_iter=max_iter, tol=tol)
    # signs: the s1 packing of the oracle's S
    assert np.array_equal(s1.cpu().numpy().view(np.uint32), oref.pack_sign(S.astype(np.float16)))
    assert abs(sigma - sig_ref) <= REL * sig_ref
    # the stopping iteration can move by one where |sigma_i - sigma_{i-1}| sits at tol * sigma
    assert abs(iters - it_ref) <= 1
    a, b = a.cpu().numpy(), b.cpu().numpy()
    assert np.max(np.abs(a - a_ref)) <= REL * np.max(np.abs(a_ref))
    assert np.max(np.abs(b - b_ref)) <= REL * np.max(np.abs(b_ref))
    assert (a > 0).all() and (b > 0).all()
    _ulp_close(g.cpu().numpy(), b_ref)
    _ulp_close(h.cpu().numpy(), a_ref)
    return s1, g, h, sigma, iters


def test_svid_4096_matches_oracle(blw, oref):
    """The OneBit 4096 x 4096 layer's initialisation from W ~ N(0, 0.02)."""
    W = synth.svid_weights(4096, 4096, seed=1)
    _, _, _, _, iters = _check(blw, oref, W)
    assert iters >= 2


def test_svid_fixed_iterations_and_ragged_shapes(blw, oref):
    """A few fixed iteration counts (tol = 0 never stops early) and shapes that
    leave partial CTAs in every pass: N not a multiple of the 8-row CTA or of
    the 128 row splits, K not a multiple of 256 columns."""
    for (N, K, it) in [(48, 384, 1), (48, 384, 3), (1040, 640, 2), (4112, 1152, 5)]:
        W = synth.svid_weights(N, K, seed=10 + N + K)
        _, _, _, _, iters = _check(blw, oref, W, max_iter=it, tol=0.0)
        assert iters == it


def test_svid_rank_one_and_signed_zeros(blw, oref):
    """An exactly rank-1 |W| (|W| = a b^T, random signs) is recovered: sigma is
    the spectral norm and a b^T = |W| to the fp32 rounding of W.  Then -0 and
    +0 entries pack as +1."""
    N, K = 64, 256
    gen = torch.Generator().manual_seed(5)
    a0 = torch.rand((N,), generator=gen, dtype=torch.float64) + 0.5
    b0 = torch.rand((K,), generator=gen, dtype=torch.float64) + 0.5
    sgn = torch.where(torch.rand((N, K), generator=gen) < 0.5, -1.0, 1.0).double()
    W = (sgn * torch.outer(a0, b0)).float()
    _, _, _, sigma, iters, a, b = blw.ob_svid(W.cuda(), return_ab=True)
    torch.cuda.synchronize()
    Wa = W.abs().double()
    assert abs(sigma - torch.linalg.matrix_norm(Wa, ord=2).item()) <= 1e-10 * sigma
    approx = torch.outer(a.cpu(), b.cpu())
    assert torch.max(torch.abs(approx - Wa)).item() <= 1e-6 * Wa.max().item()
    assert iters <= 3
    W[0, :8] = 0.0
    W[1, :8] = -0.0
    s1, _, _, _, _ = _check(blw, oref, W)
    words = s1.cpu().numpy().view(np.uint32)
    assert (words[0, 0] & 0xff) == 0xff and (words[1, 0] & 0xff) == 0xff


def test_svid_then_onebit_layer(blw, oref):
    """The device SVID feeds ob_linear directly: y matches the oracle's dense
    x (S (.) h g^T)^T with the device's g, h (the order swap)."""
    N, K = 1024, 2048
    W = synth.svid_weights(N, K, seed=77)
    s1, g, h, _, _ = blw.ob_svid(W.cuda())
    x = synth.activations(4, K, seed=78).cuda()
    y = blw.ob_linear(x, s1, g, h)
    torch.cuda.synchronize()
    S = np.where(W.numpy() < 0, -1.0, 1.0)
    dense = S * np.outer(h.cpu().numpy().astype(np.float64), g.cpu().numpy().astype(np.float64))
    ref = x.cpu().numpy().astype(np.float64) @ dense.T
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    assert np.max(err / np.max(np.abs(ref), axis=1, keepdims=True)) <= 2e-3


def test_svid_rejects_non_finite(blw):
    W = synth.svid_weights(32, 128, seed=3)
    W[5, 7] = float("inf")
    with pytest.raises(blw.BitLinearError, match="INVALID_VALUE"):
        blw.ob_svid(W.cuda())
    W[5, 7] = float("nan")
    with pytest.raises(blw.BitLinearError, match="INVALID_VALUE"):
        blw.ob_svid(W.cuda())
