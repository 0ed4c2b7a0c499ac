"""Pins for the oracle: each test checks it against something other than itself.

What pins what:
* fp16 conversion   -> numpy's IEEE binary16 conversion (library routine);
* packing           -> hand-packed golden words (tests/golden/), round trips, and the
                       OneBit page's 4096x4096 storage example;
* activation quant  -> a hand-computed token (golden) plus the invariants that the
                       BitNet b1.58 page's symmetric per-token range implies;
* ternary contraction -> numpy int64 matmul of the unpacked weights, closed forms
                       (all-ones, all-zeros, all-minus-ones), and every 3^8 pattern;
* BitLinear output  -> the fp64 value of acc * s * w_scale within fp16/fp32 rounding;
* OneBit layer      -> the order-swap identity against a dense fp64 matmul;
* SVID              -> the exact Frobenius identity, Eckart-Young against
                       numpy.linalg.svd, and Perron-Frobenius positivity.
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _golden(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, val = line.split(":", 1)
            out[key.strip()] = val.split()
    return out


# ---------------------------------------------------------------- fp16 -----

def test_half_to_double_matches_numpy_for_every_pattern(oref):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oref.half_to_double(b) for b in bits])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(got[np.isinf(ref)], ref[np.isinf(ref)])


def test_float_to_half_matches_numpy_round_to_nearest_even(oref):
    rng = np.random.default_rng(7)
    vals = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * np.float32(3.0),
        (rng.standard_normal(5000) * 1e-5).astype(np.float32),      # subnormal range
        (rng.standard_normal(2000) * 3e4).astype(np.float32),       # near overflow
        np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, -65520.0, 6.1035156e-05,
                  5.9604645e-08, 2.9802322e-08, 2.9802326e-08, 1.0009766, 1.00048828125,
                  1.00146484375, 2049.0, 2051.0], dtype=np.float32),
    ])
    # ties: values exactly halfway between two halves
    ties = (np.arange(1024, 2048, dtype=np.float32) + np.float32(0.5)) * np.float32(2.0 ** -10)
    vals = np.concatenate([vals, ties, -ties])
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float16).view(np.uint16)
    got = np.array([oref.float_to_half(v) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, ref)


# -------------------------------------------------------------- packing ----

def test_pack_ternary_golden_word(oref):
    g = _golden("pack_ternary_1x16.txt")
    t = np.array([int(v) for v in g["t"]], dtype=np.int8).reshape(1, 16)
    word = int(g["word"][0], 16)
    assert oref.pack_ternary(t)[0, 0] == word


def test_pack_sign_golden_word(oref):
    g = _golden("pack_sign_1x32.txt")
    w = np.array([float(v) for v in g["w"]], dtype=np.float16).reshape(1, 32)
    assert np.signbit(w[0, 2])  # the fixture's -0.0 survives parsing
    assert oref.pack_sign(w)[0, 0] == int(g["word"][0], 16)


def _unpack_ternary(w2, K):
    # independent decode: little-endian bytes, four 2-bit fields per byte
    b = w2.view(np.uint8).reshape(w2.shape[0], -1)
    fields = np.stack([(b >> (2 * i)) & 3 for i in range(4)], axis=-1).reshape(w2.shape[0], K)
    return fields.astype(np.int16) - 1


def _unpack_sign(s1, K):
    b = s1.view(np.uint8).reshape(s1.shape[0], -1)
    return np.unpackbits(b, axis=1, bitorder="little")[:, :K].astype(np.int8) * 2 - 1


def test_pack_ternary_round_trip(oref):
    rng = np.random.default_rng(1)
    w = rng.integers(-1, 2, size=(37, 320)).astype(np.int8)
    w2 = oref.pack_ternary(w)
    assert w2.shape == (37, 20) and w2.dtype == np.uint32
    assert np.array_equal(_unpack_ternary(w2, 320), w)
    assert not np.any(_unpack_ternary(w2, 320) == 2)   # code 3 is never written


def test_pack_ternary_rejects_values_outside_ternary(oref):
    w = np.zeros((2, 16), dtype=np.int8)
    w[1, 5] = 2
    with pytest.raises(oref.OracleError):
        oref.pack_ternary(w)


def test_pack_sign_round_trip_and_zero_is_plus_one(oref):
    rng = np.random.default_rng(2)
    w = rng.standard_normal((19, 256)).astype(np.float16)
    w[3, :17] = 0
    w[4, :9] = np.float16(-0.0)
    s = _unpack_sign(oref.pack_sign(w), 256)
    expect = np.where(w.astype(np.float32) < 0, -1, 1)
    assert np.array_equal(s, expect)
    assert np.all(s[3, :17] == 1) and np.all(s[4, :9] == 1)


def test_onebit_storage_worked_example_4096(oref):
    """OneBit page, "1. 新的 1bit 结构": a 4096x4096 layer stores a 1-bit matrix and two
    4096x1 fp16 vectors: 16,908,288 bits over 16,785,408 parameters (~1.0073 bit/param)."""
    N = K = 4096
    rng = np.random.default_rng(3)
    w = np.where(rng.integers(0, 2, size=(N, K)) == 1, 1.0, -1.0).astype(np.float16)
    s1 = oref.pack_sign(w)
    g = np.ones(K, dtype=np.float16)
    h = np.ones(N, dtype=np.float16)
    bits = 8 * (s1.nbytes + g.nbytes + h.nbytes)
    assert s1.nbytes == 2_097_152
    assert bits == 16_908_288 == oref.onebit_bits(N, K)
    params = N * K + N + K
    assert params == 16_785_408 == oref.onebit_params(N, K)
    assert round(bits / params, 4) == 1.0073


# ----------------------------------------------------- activation quant ----

def test_act_quant_golden_token(oref):
    g = _golden("act_quant_1x8.txt")
    x = np.array([float(v) for v in g["x"]], dtype=np.float16).reshape(1, 8)
    q, s = oref.quant_act(x)
    assert q[0].tolist() == [int(v) for v in g["q"]]
    assert s[0] == np.float32(float(g["s"][0]))


def test_act_quant_invariants(oref):
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((64, 512)) * rng.uniform(0.01, 50, size=(64, 1))).astype(np.float16)
    x[5] = 0                                   # an all-zero token
    x[6, 17] = np.float16(-30000)              # a dominant negative outlier
    q, s = oref.quant_act(x)
    xf = x.astype(np.float64)
    amax = np.abs(xf).max(axis=1)
    assert np.all(np.abs(q.astype(np.int32)) <= 127)
    assert np.all(q[5] == 0) and s[5] == 0
    for m in range(64):
        if amax[m] == 0:
            continue
        am = np.argmax(np.abs(xf[m]))
        assert q[m, am] == (127 if xf[m, am] > 0 else -127)
        nz = q[m] != 0
        assert np.all(np.sign(q[m][nz]) == np.sign(xf[m][nz]))
        # q is the nearest integer to x*127/amax (fp32 scale rounding slack only)
        assert np.max(np.abs(xf[m] * 127.0 / amax[m] - q[m])) <= 0.5 + 1e-4
        assert abs(s[m] * 127.0 / amax[m] - 1.0) < 2e-7
    assert q[6, 17] == -127


def test_act_quant_rounds_fp32_product_then_to_integer(oref):
    """q = rne(fp32(x * fp32(127/amax))): the product is rounded to fp32 first
    (the reading of the BitNet b1.58 page's quantiser: scale by the fp32 inverse,
    then round half to even).  For amax = 4.6328125 and x = amax/2 the exact
    product 127/2 * (1 + delta) lies just below 63.5, rounds to 63.5 in fp32 and
    then to 64; a single rounding of the exact product would give 63."""
    amax = np.float16(4.6328125)
    x = np.zeros((1, 16), dtype=np.float16)
    x[0, 0] = amax
    x[0, 3] = np.float16(amax / 2)
    x[0, 9] = np.float16(-amax / 2)
    inv = np.float32(127.0) / np.float32(amax)
    exact = float(np.float64(x[0, 3]) * np.float64(inv))
    assert 63.49 < exact < 63.5                        # below the tie in exact arithmetic
    assert np.float32(np.float32(x[0, 3]) * inv) == np.float32(63.5)
    q, s = oref.quant_act(x)
    assert q[0, 0] == 127 and q[0, 3] == 64 and q[0, 9] == -64


# ------------------------------------------------- ternary contraction -----

def _bitlinear_case(oref, M, K, N, seed, w=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float16)
    if w is None:
        w = rng.integers(-1, 2, size=(N, K)).astype(np.int8)
    y, acc = oref.ternary_linear(x, oref.pack_ternary(w), 0.02)
    q, s = oref.quant_act(x)
    return x, w, q, s, y, acc


def test_ternary_acc_matches_int64_matmul(oref):
    x, w, q, s, y, acc = _bitlinear_case(oref, 7, 384, 48, seed=5)
    ref = q.astype(np.int64) @ w.astype(np.int64).T
    assert np.array_equal(acc.astype(np.int64), ref)


@pytest.mark.parametrize("fill", [1, 0, -1])
def test_ternary_acc_closed_forms(oref, fill):
    K, N = 256, 16
    w = np.full((N, K), fill, dtype=np.int8)
    x, w, q, s, y, acc = _bitlinear_case(oref, 3, K, N, seed=6, w=w)
    rowsum = q.astype(np.int64).sum(axis=1)
    assert np.array_equal(acc, np.repeat((fill * rowsum)[:, None], N, axis=1))


def test_ternary_acc_exhaustive_patterns_k8(oref):
    """Every one of the 3^8 ternary patterns on the first 8 inputs (rest zero)."""
    pats = np.array(np.meshgrid(*[[-1, 0, 1]] * 8, indexing="ij")).reshape(8, -1).T
    N = pats.shape[0]
    w = np.zeros((N, 16), dtype=np.int8)
    w[:, :8] = pats
    x = np.array([[3.0, -1.0, 0.5, 2.0, -2.5, 1.5, -0.75, 0.25] + [0.1] * 8], dtype=np.float16)
    y, acc = oref.ternary_linear(x, oref.pack_ternary(w), 1.0)
    q, s = oref.quant_act(x)
    brute = [sum(int(q[0, k]) * int(w[n, k]) for k in range(8)) for n in range(N)]
    assert acc[0].tolist() == brute


def test_bitlinear_output_within_rounding_of_exact(oref):
    x, w, q, s, y, acc = _bitlinear_case(oref, 9, 512, 64, seed=8)
    exact = acc.astype(np.float64) * s.astype(np.float64)[:, None] * np.float64(np.float32(0.02))
    err = np.abs(y.astype(np.float64) - exact)
    # fp16 rounding (2^-11 relative, or half the subnormal step) + two fp32 roundings
    bound = np.maximum(np.abs(exact) * (2.0 ** -11 + 2.0 ** -22), 2.0 ** -25)
    assert np.all(err <= bound)
    assert np.max(err) / np.max(np.abs(exact)) <= 1e-3


def test_bitlinear_all_zero_token_gives_zero(oref):
    x = np.zeros((2, 128), dtype=np.float16)
    x[1, 3] = 1.0
    w = np.ones((16, 128), dtype=np.int8)
    y, acc = oref.ternary_linear(x, oref.pack_ternary(w), 0.02)
    assert np.all(acc[0] == 0) and np.all(y[0] == 0)
    assert np.all(acc[1] == 127)


# ---------------------------------------------------------------- OneBit ---

def test_onebit_order_swap_identity(oref):
    """OneBit page, "2. 基于 SVID 初始化量化模型": swapping the order of operations
    makes ((x*g) S^T) * h equal x (S * h g^T)^T."""
    rng = np.random.default_rng(9)
    M, K, N = 5, 320, 40
    x = rng.standard_normal((M, K)).astype(np.float16)
    S = np.where(rng.integers(0, 2, size=(N, K)) == 1, 1.0, -1.0)
    g = ((rng.uniform(size=K) + 0.5) * 0.02).astype(np.float16)
    h = ((rng.uniform(size=N) + 0.5) * 0.02).astype(np.float16)
    y, z = oref.ob_linear(x, oref.pack_sign(S.astype(np.float16)), g, h)
    Wd = S * np.outer(h.astype(np.float64), g.astype(np.float64))
    ref = x.astype(np.float64) @ Wd.T
    assert np.max(np.abs(z - ref)) <= 1e-12 * np.max(np.abs(ref))
    assert np.array_equal(y, ref.astype(np.float16))  # single rounding of the same value


def test_onebit_brute_force_tiny(oref):
    rng = np.random.default_rng(10)
    M, K, N = 2, 32, 3
    x = rng.standard_normal((M, K)).astype(np.float16)
    Wf = rng.standard_normal((N, K)).astype(np.float16)
    g = rng.uniform(0.5, 1.5, size=K).astype(np.float16)
    h = rng.uniform(0.5, 1.5, size=N).astype(np.float16)
    y, z = oref.ob_linear(x, oref.pack_sign(Wf), g, h)
    for m in range(M):
        for n in range(N):
            tot = 0.0
            for k in range(K):
                sgn = -1.0 if float(Wf[n, k]) < 0 else 1.0
                tot += float(x[m, k]) * float(g[k]) * sgn
            assert abs(z[m, n] - tot * float(h[n])) <= 1e-12 * (1 + abs(tot))


# ------------------------------------------------------------------ SVID ---

def test_svid_rank1_identities(oref):
    rng = np.random.default_rng(11)
    N, K = 96, 160
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[0, 0] = 0.0
    S, a, b, sigma, iters = oref.svid(W)
    Wd = W.astype(np.float64)
    assert np.array_equal(S, np.where(Wd < 0, -1, 1).astype(np.int8))
    assert np.all(a > 0) and np.all(b > 0)                    # Perron-Frobenius
    approx = S * np.outer(a, b)
    lhs = np.linalg.norm(Wd - approx)
    rhs = np.linalg.norm(np.abs(Wd) - np.outer(a, b))
    assert abs(lhs - rhs) <= 1e-12 * np.linalg.norm(Wd)        # S*S = 1 element-wise
    sv = np.linalg.svd(np.abs(Wd), compute_uv=False)
    assert abs(sigma - sv[0]) <= 1e-9 * sv[0]
    eckart_young = np.sqrt(max(np.sum(sv ** 2) - sv[0] ** 2, 0.0))
    assert abs(rhs - eckart_young) <= 1e-7 * np.linalg.norm(Wd)
    assert iters < 1000


def test_svid_drives_onebit_layer_by_order_swap(oref):
    """SVID's factors used as h = a and g = b make the 1-bit layer reproduce
    x (S * a b^T)^T (with the factors rounded to fp16 as the layer stores them)."""
    rng = np.random.default_rng(12)
    N, K, M = 64, 128, 3
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    S, a, b, sigma, _ = oref.svid(W)
    g = b.astype(np.float16)
    h = a.astype(np.float16)
    x = rng.standard_normal((M, K)).astype(np.float16)
    y, z = oref.ob_linear(x, oref.pack_sign(W.astype(np.float16)), g, h)
    Wd = S * np.outer(h.astype(np.float64), g.astype(np.float64))
    ref = x.astype(np.float64) @ Wd.T
    assert np.max(np.abs(z - ref)) <= 1e-12 * np.max(np.abs(ref))


def test_openmp_build_gives_identical_results(oref):
    """The all-cores oracle build (output rows spread over OpenMP threads) is
    the same scalar loop per output: bit-identical y, accumulators and z."""
    from bit_weight_linear_b200 import synth
    x = synth.activations(3, 640, seed=77, outlier_frac=0.01).numpy()
    w2 = oref.pack_ternary(synth.ternary_weights(272, 640, seed=78).numpy())
    y1, a1 = oref.ternary_linear(x, w2, 0.02)
    y2, a2 = oref.ternary_linear(x, w2, 0.02, parallel=True)
    assert np.array_equal(a1, a2) and np.array_equal(y1.view(np.uint16), y2.view(np.uint16))
    s1 = oref.pack_sign(synth.sign_weights(96, 640, seed=79).numpy())
    g = synth.value_vector(640, seed=80).numpy()
    h = synth.value_vector(96, seed=81).numpy()
    _, z1 = oref.ob_linear(x, s1, g, h)
    _, z2 = oref.ob_linear(x, s1, g, h, parallel=True)
    assert np.array_equal(z1, z2)


# ------------------------------------------------ RMSNorm and SwiGLU -----

def _golden_rows(name):
    rows = {}
    for line in open(os.path.join(os.path.dirname(__file__), "golden", name)):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            rows[k] = v
    return rows


def test_rmsnorm_hand_worked_token(oref):
    g = _golden_rows("rmsnorm_3_4.txt")
    x = np.array([[float(v) for v in g["x"]]], dtype=np.float16)
    y = oref.rmsnorm(x, np.ones(2, dtype=np.float16), 0.0)
    assert [int(b) for b in y.view(np.uint16)[0]] == [int(v, 16) for v in g["y_bits"]]


@pytest.mark.parametrize("K", [64, 640, 4096])
def test_rmsnorm_against_exactly_rounded_sum(oref, K):
    """The definition evaluated independently: math.fsum is the exactly rounded
    sum of the squares (each exact in fp64 for fp16 inputs), then the same
    fp64 steps in numpy, then numpy's fp16 rounding."""
    import math
    rng = np.random.default_rng(K)
    x = (rng.standard_normal((3, K)) * np.array([[1.0], [1e-3], [300.0]])).astype(np.float16)
    x[1, 5] = np.float16(6e-8)          # a subnormal
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float16)
    eps = 1e-6
    y = oref.rmsnorm(x, gamma, eps)
    for m in range(3):
        xd = x[m].astype(np.float64)
        ss = math.fsum(float(v) * float(v) for v in xd)
        r = 1.0 / math.sqrt(ss / K + eps)
        ref = ((xd * r) * gamma.astype(np.float64)).astype(np.float16)
        assert np.array_equal(y[m].view(np.uint16), ref.view(np.uint16)), m


def test_rmsnorm_scale_invariance_and_unit_rms(oref):
    """With eps = 0 the output does not change when x is scaled by a power of
    two (the mean square scales by its square, exactly); with gamma = 1 the
    output's mean square is 1 up to fp16 rounding."""
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 1024)).astype(np.float16)
    one = np.ones(1024, dtype=np.float16)
    y = oref.rmsnorm(x, one, 0.0)
    for j in (1, 3):
        xs = (x.astype(np.float64) * 2.0 ** j).astype(np.float16)
        assert np.array_equal(xs.astype(np.float64), x.astype(np.float64) * 2.0 ** j)  # exact scaling
        ys = oref.rmsnorm(xs, one, 0.0)
        assert np.array_equal(ys.view(np.uint16), y.view(np.uint16))
    ms = np.mean(y.astype(np.float64) ** 2, axis=1)
    assert np.all(np.abs(ms - 1.0) < 2e-3)


def test_swiglu_identities(oref):
    """silu(a) - silu(-a) = a exactly (1/(1+e^-a) + 1/(1+e^a) = 1), silu(0) = 0,
    silu(a) -> a for large a and -> 0 for very negative a; b scales the output."""
    a = np.linspace(-12, 12, 481).astype(np.float16)
    one = np.ones_like(a)
    yp = oref.swiglu(a, one).astype(np.float64)
    yn = oref.swiglu(-a, one).astype(np.float64)
    diff = yp - yn
    # each side carries one fp16 rounding: at most half an fp16 spacing of |silu|
    tol = 2.0 ** -10 * np.maximum(np.abs(yp), np.abs(yn)) + 2.0 ** -24
    assert np.all(np.abs(diff - a.astype(np.float64)) <= tol)
    assert oref.swiglu(np.zeros(1, np.float16), np.ones(1, np.float16))[0] == 0
    big = np.array([30.0, -30.0], dtype=np.float16)
    yb = oref.swiglu(big, np.ones(2, np.float16))
    assert yb[0] == np.float16(30.0) and abs(float(yb[1])) < 1e-10
    b = np.full_like(a, 2.0)
    assert np.array_equal(oref.swiglu(a, b).astype(np.float64), 2 * oref.swiglu(a, one).astype(np.float64))


# ---- BiLLM binary residual approximation (oracle.billm_binarize / billm_linear)

def _pad32(rows):
    """Pad int8 +-1 rows to 32 columns with +1 (zero x there) for the s1 packing."""
    out = np.ones((rows.shape[0], 32), dtype=np.int8)
    out[:, :rows.shape[1]] = rows
    return out


def test_billm_hand_worked_rows(oref):
    g = _golden_rows("billm_residual_2x4.txt")
    W = np.array([[float(v) for v in g["w0"]], [float(v) for v in g["w1"]]], dtype=np.float32)
    Bo, Br, ao, ar = oref.billm_binarize(W)
    assert Bo.tolist() == [[int(v) for v in g["bo0"]], [int(v) for v in g["bo1"]]]
    assert Br.tolist() == [[int(v) for v in g["br0"]], [int(v) for v in g["br1"]]]
    assert ao.tolist() == [float(v) for v in g["alpha_o"]]
    assert ar.tolist() == [float(v) for v in g["alpha_r"]]
    assert (ao[0] * Bo[0] + ar[0] * Br[0]).tolist() == [float(v) for v in g["approx0"]]
    # the linear layer on those planes (zero-padded to one 32-bit word)
    x = np.zeros((1, 32), dtype=np.float16)
    x[0, :4] = [float(v) for v in g["x"]]
    bo1 = oref.pack_sign(_pad32(Bo).astype(np.float16))
    br1 = oref.pack_sign(_pad32(Br).astype(np.float16))
    y, z = oref.billm_linear(x, bo1, br1, ao.astype(np.float16), ar.astype(np.float16))
    assert z[0].tolist() == [float(v) for v in g["y"]]


def test_billm_residual_never_worse_and_scales_optimal(oref):
    """The page's property: the residual approximation's error is at most that
    of plain binarisation.  And each alpha is the least-squares scale of its
    sign plane: moving it either way increases the row's error."""
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32)
    W[3] = rng.laplace(size=512).astype(np.float32)            # heavier tails
    Bo, Br, ao, ar = oref.billm_binarize(W)
    Wd = W.astype(np.float64)
    e1 = np.sum((Wd - ao[:, None] * Bo) ** 2, axis=1)
    e2 = np.sum((Wd - ao[:, None] * Bo - ar[:, None] * Br) ** 2, axis=1)
    assert (e2 <= e1).all() and (e2 < 0.6 * e1).all()
    assert np.array_equal(Bo, np.where(W < 0, -1, 1))
    R = Wd - ao[:, None] * Bo
    assert np.array_equal(Br, np.where(R < 0, -1, 1))
    for f in (1 - 1e-3, 1 + 1e-3):
        assert (np.sum((Wd - f * ao[:, None] * Bo) ** 2, axis=1) > e1).all()
        assert (np.sum((R - f * ar[:, None] * Br) ** 2, axis=1) >
                np.sum((R - ar[:, None] * Br) ** 2, axis=1)).all()


def test_billm_linear_against_dense_and_special_cases(oref):
    """z equals the dense fp64 product with alpha_o B_o + alpha_r B_r; with
    B_r = B_o it is (alpha_o + alpha_r) x B_o^T; with alpha_r = 0 it is the
    OneBit layer with g = 1 and h = alpha_o."""
    rng = np.random.default_rng(11)
    M, K, N = 3, 256, 48
    x = rng.standard_normal((M, K)).astype(np.float16)
    Bo = np.where(rng.random((N, K)) < 0.5, -1, 1).astype(np.int8)
    Br = np.where(rng.random((N, K)) < 0.5, -1, 1).astype(np.int8)
    ao = rng.uniform(0.01, 0.03, N).astype(np.float16)
    ar = rng.uniform(0.002, 0.01, N).astype(np.float16)
    bo1, br1 = oref.pack_sign(Bo.astype(np.float16)), oref.pack_sign(Br.astype(np.float16))
    y, z = oref.billm_linear(x, bo1, br1, ao, ar)
    dense = ao.astype(np.float64)[:, None] * Bo + ar.astype(np.float64)[:, None] * Br
    ref = x.astype(np.float64) @ dense.T
    assert np.max(np.abs(z - ref)) <= 1e-12 * np.max(np.abs(ref))
    assert np.array_equal(y, ref.astype(np.float16)) or \
        np.max(np.abs(y.astype(np.float64) - ref)) <= 2.0 ** -10 * np.max(np.abs(ref))
    _, z_same = oref.billm_linear(x, bo1, bo1, ao, ar)
    ref_same = (ao.astype(np.float64) + ar.astype(np.float64)) * (x.astype(np.float64) @ Bo.T.astype(np.float64))
    assert np.max(np.abs(z_same - ref_same)) <= 1e-12 * np.max(np.abs(ref_same))
    _, z_zero = oref.billm_linear(x, bo1, br1, ao, np.zeros(N, dtype=np.float16))
    _, z_ob = oref.ob_linear(x, bo1, np.ones(K, dtype=np.float16), ao)
    assert np.max(np.abs(z_zero - z_ob)) <= 1e-12 * np.max(np.abs(z_ob))
