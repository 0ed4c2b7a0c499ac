"""Host-side check of the OneBit fixed-point image the CUDA kernels use (no GPU).

The kernels contract a per-token integer image of x*g instead of the floating
values: X = rne(x*g * rn((2^22 - 1) / amax')), amax' = max_k |x*g| (fp32, the
products are exact), then sum_k X*S exactly in integers and one fp32 scale
by amax' / (2^22 - 1).  The image's error is at most amax' / (2 (2^22 - 1))
per element, so a token whose largest |x*g| dwarfs the rest (one outlier
activation) is where the image is coarsest relative to the other elements.

This restates that arithmetic in numpy (not the CUDA code) and checks it
against the fp64 oracle on such tokens, at the longest rows the layer takes
(K = 65536) and the 13B-shaped down layer, with margin under the 2e-3 bar of
the OneBit statement (OneBit page, "1. 新的 1bit 结构": only g and h are FP16,
the activations are not quantised; the bar is max|y - y_ref| / max|y_ref|)."""
import numpy as np
import pytest

from bit_weight_linear_b200 import synth

IMG_MAX = np.float32(4194303.0)


def image_layer(x16, s1_bits, g16, h16):
    """fp32 image arithmetic of the kernels, in numpy: returns z*h in fp64."""
    xg = x16.astype(np.float32) * g16.astype(np.float32)      # exact in fp32
    amax = np.max(np.abs(xg), axis=1).astype(np.float32)
    inv = np.where(amax > 0, IMG_MAX / np.where(amax > 0, amax, 1), 0).astype(np.float32)
    X = np.rint((xg * inv[:, None]).astype(np.float32)).astype(np.int64)
    assert np.max(np.abs(X)) <= 4194303
    Z = X @ s1_bits.T.astype(np.int64)                         # exact
    step = (amax / IMG_MAX).astype(np.float32)
    z = (step[:, None] * Z.astype(np.float32)).astype(np.float32)
    return z.astype(np.float64) * h16.astype(np.float64)[None, :]


@pytest.mark.parametrize("K,N", [(13824, 64), (65536, 32)])
@pytest.mark.parametrize("val", [2000.0, -60000.0])
def test_image_meets_the_bar_on_outlier_tokens(oref, K, N, val):
    M = 3
    x = synth.activations(M, K, seed=9_000 + K).numpy()
    x[0, 5] = val
    x[2, K - 1] = -val / 7
    w = synth.sign_weights(N, K, seed=9_001 + K).numpy()
    g = synth.value_vector(K, seed=9_002).numpy()
    h = synth.value_vector(N, seed=9_003).numpy()
    s1 = oref.pack_sign(w)
    _, z_ref = oref.ob_linear(x, s1, g, h)
    signs = np.where(w >= 0, 1, -1).astype(np.int64)
    z = image_layer(x, signs, g, h)
    for m in range(M):
        err = np.max(np.abs(z[m] - z_ref[m])) / np.max(np.abs(z_ref[m]))
        # the image's error alone; fp16 rounding of y adds at most 2^-11
        assert err <= 1e-4, (m, err)


def test_a_16_bit_image_would_miss_the_bar():
    """The same arithmetic with a 16-bit image (2^15 - 129 levels) fails the
    2e-3 bar on an outlier token at K = 13824: the reason for the wider image."""
    K, N = 13824, 256
    x = synth.activations(1, K, seed=9_100).numpy()
    x[0, 17] = 2000.0
    w = synth.sign_weights(N, K, seed=9_101).numpy()
    g = synth.value_vector(K, seed=9_102).numpy()
    h = synth.value_vector(N, seed=9_103).numpy()
    xg = x.astype(np.float32) * g.astype(np.float32)
    amax = np.float32(np.max(np.abs(xg)))
    X = np.rint(xg * (np.float32(32639.0) / amax)).astype(np.int64)
    signs = np.where(w >= 0, 1, -1).astype(np.int64)
    z16 = (X @ signs.T).astype(np.float64) * float(amax / np.float32(32639.0)) * h.astype(np.float64)
    exact = (xg.astype(np.float64) @ signs.T.astype(np.float64)) * h.astype(np.float64)
    assert np.max(np.abs(z16 - exact)) / np.max(np.abs(exact)) > 2e-3
