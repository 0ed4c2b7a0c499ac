"""GPU parity: the CUDA path (through the C ABI) against the oracle on the same
seeded inputs.

Bars (from the statement of the two layer forms):
* packed bytes, int8 activations, fp32 token scales and int32 accumulators:
  bit-exact;
* BitLinear fp16 output: max|y_gpu - y_ref| / max|y_ref| <= 1e-3 (the GPU
  evaluates the same fp32 sequence, so it is also checked bit-exact);
* OneBit fp16 output: max|y_gpu - y_ref| / max|y_ref| <= 2e-3 against the fp64
  oracle.
"""
import numpy as np
import pytest
import torch

from bit_weight_linear_b200 import synth

pytestmark = pytest.mark.gpu

BL_TOL = 1e-3
OB_TOL = 2e-3


@pytest.fixture(scope="module")
def blw():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_linear_b200 import build
    build.build()
    import bit_weight_linear_b200 as m
    return m


def _np_u32(t):
    return t.cpu().numpy().view(np.uint32)


def _rel_err(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    den = np.max(np.abs(b))
    return float(np.max(np.abs(a - b)) / (den if den > 0 else 1.0))


# ------------------------------------------------------------- packers -----

@pytest.mark.parametrize("N,K", [(16, 128), (48, 384), (272, 640), (4096, 4096)])
def test_pack_ternary_bytes_identical(blw, oref, N, K):
    w = synth.ternary_weights(N, K, seed=N + K)
    w2 = blw.bl_pack_ternary(w.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_np_u32(w2), oref.pack_ternary(w.numpy()))


def test_pack_ternary_rejects_invalid(blw):
    w = torch.zeros((16, 128), dtype=torch.int8)
    w[7, 33] = 2
    with pytest.raises(blw.BitLinearError) as e:
        blw.bl_pack_ternary(w.cuda())
    assert e.value.status == 4
    w[7, 33] = -128
    with pytest.raises(blw.BitLinearError):
        blw.bl_pack_ternary(w.cuda())
    w[7, 33] = 1
    blw.bl_pack_ternary(w.cuda())   # the error word is cleared per call


@pytest.mark.parametrize("N,K", [(16, 128), (48, 384), (4096, 4096)])
def test_pack_sign_bytes_identical(blw, oref, N, K):
    w = synth.svid_weights(N, K, seed=3).to(torch.float16)
    w[0, :40] = 0.0
    w[1, :40] = -0.0
    s1 = blw.ob_pack_sign(w.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_np_u32(s1), oref.pack_sign(w.numpy()))


def test_pack_sign_rejects_nan(blw):
    w = torch.ones((16, 128), dtype=torch.float16)
    w[3, 3] = float("nan")
    with pytest.raises(blw.BitLinearError) as e:
        blw.ob_pack_sign(w.cuda())
    assert e.value.status == 4


# ------------------------------------------------------ activation quant ---

@pytest.mark.parametrize("M,K", [(1, 128), (3, 384), (77, 4096), (5, 28672)])
def test_quant_act_bit_exact(blw, oref, M, K):
    x = synth.activations(M, K, seed=M * 7 + K, outlier_frac=0.01)
    if M > 2:
        x[1] = 0.0                       # all-zero token
        x[2, 5] = -60000.0               # dominant negative outlier
    q, s = blw.bl_quant_act(x.cuda())
    torch.cuda.synchronize()
    q_ref, s_ref = oref.quant_act(x.numpy())
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


# ----------------------------------------------------------- BitLinear -----

TERNARY_SHAPES = [
    (1, 128, 16), (1, 384, 48), (3, 640, 272), (8, 4096, 4096),      # the M=8 4096^2 layer
    (9, 384, 64), (17, 1152, 96), (40, 256, 32), (100, 768, 48), (1, 11008, 64),
]


@pytest.mark.parametrize("M,K,N", TERNARY_SHAPES)
def test_ternary_linear_parity(blw, oref, M, K, N):
    x = synth.activations(M, K, seed=11 + M + K + N)
    w = synth.ternary_weights(N, K, seed=12 + M + K + N)
    w2 = oref.pack_ternary(w.numpy())
    y, acc = blw.bl_ternary_linear(x.cuda(), torch.from_numpy(w2.view(np.int32)).cuda(), 0.02,
                                   return_acc=True)
    torch.cuda.synchronize()
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), w2, 0.02)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    yg = y.cpu().numpy()
    assert _rel_err(yg, y_ref) <= BL_TOL
    assert np.array_equal(yg.view(np.uint16), y_ref.view(np.uint16))


def test_ternary_linear_special_weights_and_zero_token(blw, oref):
    M, K, N = 4, 512, 48
    x = synth.activations(M, K, seed=21)
    x[2] = 0.0
    w = torch.zeros((N, K), dtype=torch.int8)
    w[:16] = 1
    w[16:32] = -1
    w2 = blw.bl_pack_ternary(w.cuda())
    y, acc = blw.bl_ternary_linear(x.cuda(), w2, 0.5, return_acc=True)
    torch.cuda.synchronize()
    q_ref, _ = oref.quant_act(x.numpy())
    rs = q_ref.astype(np.int64).sum(axis=1)
    a = acc.cpu().numpy()
    assert np.array_equal(a[:, :16], np.repeat(rs[:, None], 16, axis=1))
    assert np.array_equal(a[:, 16:32], -np.repeat(rs[:, None], 16, axis=1))
    assert np.all(a[:, 32:] == 0)
    assert np.all(y.cpu().numpy()[2] == 0)


def test_ternary_linear_deterministic(blw):
    M, K, N = 8, 4096, 512
    x = synth.activations(M, K, seed=31).cuda()
    w2 = blw.bl_pack_ternary(synth.ternary_weights(N, K, seed=32).cuda())
    y1, a1 = blw.bl_ternary_linear(x, w2, 0.02, return_acc=True)
    y2, a2 = blw.bl_ternary_linear(x, w2, 0.02, return_acc=True)
    torch.cuda.synchronize()
    assert torch.equal(a1, a2) and torch.equal(y1.view(torch.int16), y2.view(torch.int16))


# --------------------------------------------------------------- OneBit ----

ONEBIT_SHAPES = [
    (1, 128, 16), (1, 384, 48), (3, 640, 272), (1, 4096, 4096), (16, 4096, 4096),
    (5, 1152, 96), (9, 256, 32), (33, 768, 48), (1, 13824, 64),
]


def _onebit_inputs(M, K, N, seed):
    x = synth.activations(M, K, seed=seed)
    ws = synth.sign_weights(N, K, seed=seed + 1)
    g = synth.value_vector(K, seed=seed + 2)
    h = synth.value_vector(N, seed=seed + 3)
    return x, ws, g, h


@pytest.mark.parametrize("M,K,N", ONEBIT_SHAPES)
def test_ob_linear_parity(blw, oref, M, K, N):
    x, ws, g, h = _onebit_inputs(M, K, N, seed=41 + M + K + N)
    s1 = oref.pack_sign(ws.numpy())
    y = blw.ob_linear(x.cuda(), torch.from_numpy(s1.view(np.int32)).cuda(), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    y_ref, z_ref = oref.ob_linear(x.numpy(), s1, g.numpy(), h.numpy())
    assert _rel_err(y.cpu().numpy(), z_ref) <= OB_TOL


def test_ob_linear_svid_initialised_layer(blw, oref):
    """A OneBit layer initialised by SVID (sign of W, rank-1 factors of |W| as h
    and g) gives the oracle's output through the CUDA path."""
    N, K, M = 256, 512, 4
    W = synth.svid_weights(N, K, seed=51).numpy()
    S, a, b, sigma, _ = oref.svid(W)
    g = torch.from_numpy(b.astype(np.float16))
    h = torch.from_numpy(a.astype(np.float16))
    x = synth.activations(M, K, seed=52)
    s1 = blw.ob_pack_sign(torch.from_numpy(W).to(torch.float16).cuda())
    y = blw.ob_linear(x.cuda(), s1, g.cuda(), h.cuda())
    torch.cuda.synchronize()
    _, z_ref = oref.ob_linear(x.numpy(), oref.pack_sign(W.astype(np.float16)), g.numpy(), h.numpy())
    assert _rel_err(y.cpu().numpy(), z_ref) <= OB_TOL


def test_ob_linear_zero_token(blw):
    M, K, N = 3, 256, 32
    x, ws, g, h = _onebit_inputs(M, K, N, seed=61)
    x[1] = 0
    y = blw.ob_linear(x.cuda(), blw.ob_pack_sign(ws.cuda()), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    assert torch.all(y[1] == 0)


# ------------------------------------------------- tensor-core prefill ------

PREFILL_TERNARY = [(33, 128, 16), (128, 4096, 512), (200, 384, 272), (512, 1024, 1024),
                   (77, 11008, 256), (300, 640, 48),
                   # 4 and 2 k-blocks per stage with a short last stage (9 and 15 blocks)
                   (40, 1152, 96), (100, 1920, 128)]


@pytest.mark.parametrize("M,K,N", PREFILL_TERNARY)
def test_ternary_prefill_parity(blw, oref, M, K, N):
    x = synth.activations(M, K, seed=71 + M + K + N, outlier_frac=0.01)
    w = synth.ternary_weights(N, K, seed=72 + M + K + N)
    w2 = oref.pack_ternary(w.numpy())
    y, acc = blw.bl_ternary_linear(x.cuda(), torch.from_numpy(w2.view(np.int32)).cuda(), 0.02,
                                   return_acc=True)
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), w2, 0.02)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    yg = y.cpu().numpy()
    assert _rel_err(yg, y_ref) <= BL_TOL
    assert np.array_equal(yg.view(np.uint16), y_ref.view(np.uint16))


PREFILL_ONEBIT = [(17, 128, 16), (64, 4096, 512), (150, 640, 272), (256, 1024, 1024),
                  (40, 640, 64)]


@pytest.mark.parametrize("M,K,N", PREFILL_ONEBIT)
def test_onebit_prefill_parity(blw, oref, M, K, N):
    x, ws, g, h = _onebit_inputs(M, K, N, seed=81 + M + K + N)
    s1 = oref.pack_sign(ws.numpy())
    y = blw.ob_linear(x.cuda(), torch.from_numpy(s1.view(np.int32)).cuda(), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    _, z_ref = oref.ob_linear(x.numpy(), s1, g.numpy(), h.numpy())
    assert _rel_err(y.cpu().numpy(), z_ref) <= OB_TOL


def test_ternary_prefill_70b_full_size_sampled_rows(blw, oref):
    """The 70B-shaped gate/up layer (K=8192, N=28672) at M=512 with 1% outlier
    channels, run whole on the GPU; the oracle recomputes 96 sampled weight rows
    for all 512 tokens (rows are independent)."""
    M, K, N = 512, 8192, 28672
    # 448 tiles: two whole-tile rounds, then a balanced round of the last 152
    assert blw.bl_ternary_workspace_bytes(M, K, N) > M * K + 1_000_000
    x = synth.activations(M, K, seed=3_000_001, outlier_frac=0.01)
    w = synth.ternary_weights(N, K, seed=3_000_008)
    y, acc = blw.bl_ternary_linear(x.cuda(), blw.bl_pack_ternary(w.cuda()), 0.02, return_acc=True)
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(5).choice(N, size=96, replace=False))
    rows[-1] = N - 1
    w2s = oref.pack_ternary(w.numpy()[rows])
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), w2s, 0.02)
    assert np.array_equal(acc.cpu().numpy()[:, rows], acc_ref)
    assert np.array_equal(y.cpu().numpy()[:, rows].view(np.uint16), y_ref.view(np.uint16))


# Shapes whose tiles leave most SMs idle in the last round on a 148-SM part, so
# the kernel shares the work out in k-stages and finishes split tiles from int32
# partials: 150 tiles of 100 tokens with two 128-k blocks per ring stage, and
# 150 ragged tiles (a 44-row token tile, an 80-column weight tile).
BALANCED_ROUND = [(100, 16384, 19200), (300, 8192, 9552)]


@pytest.mark.parametrize("M,K,N", BALANCED_ROUND)
def test_ternary_prefill_balanced_round(blw, oref, M, K, N):
    """The integer accumulators of split tiles must still be exact.  Sampled
    weight rows (first and last included), all tokens."""
    # the workspace carries the split scratch only when the plan uses it
    assert blw.bl_ternary_workspace_bytes(M, K, N) > M * K + 1_000_000
    x = synth.activations(M, K, seed=3_100_001 + M, outlier_frac=0.01)
    w = synth.ternary_weights(N, K, seed=3_100_002 + M)
    y, acc = blw.bl_ternary_linear(x.cuda(), blw.bl_pack_ternary(w.cuda()), 0.02, return_acc=True)
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    rows = np.sort(np.random.default_rng(7).choice(N, size=128, replace=False))
    rows[0], rows[-1] = 0, N - 1
    w2s = oref.pack_ternary(w.numpy()[rows])
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), w2s, 0.02)
    assert np.array_equal(acc.cpu().numpy()[:, rows], acc_ref)
    assert np.array_equal(y.cpu().numpy()[:, rows].view(np.uint16), y_ref.view(np.uint16))


# Small token counts on the tensor-core path (ternary from M = 9, OneBit from
# M = 5): 32-row activation tiles with four 128-k blocks per ring stage.  The
# 13824-long layers have 40 tiles, which the kernel shares out over all SMs.
# Large layers are checked on 128 sampled weight rows (first and last
# included, so every tile is likely hit), small ones whole.
SMALL_M_TERNARY = [(9, 13824, 5120), (16, 13824, 5120), (12, 4096, 4096), (9, 2048, 1024)]
SMALL_M_ONEBIT = [(3, 13824, 5120), (4, 5120, 13824), (5, 13824, 5120), (8, 13824, 5120), (8, 5120, 13824)]


def _sample_rows(N, seed):
    if N <= 4096:
        return np.arange(N)
    rows = np.sort(np.random.default_rng(seed).choice(N, size=128, replace=False))
    rows[0], rows[-1] = 0, N - 1
    return rows


@pytest.mark.parametrize("M,K,N", SMALL_M_TERNARY)
def test_ternary_prefill_small_token_counts(blw, oref, M, K, N):
    x = synth.activations(M, K, seed=3_200_000 + M + N, outlier_frac=0.01)
    w = synth.ternary_weights(N, K, seed=3_200_001 + M + N)
    y, acc = blw.bl_ternary_linear(x.cuda(), blw.bl_pack_ternary(w.cuda()), 0.02, return_acc=True)
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    rows = _sample_rows(N, seed=M)
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), oref.pack_ternary(w.numpy()[rows]), 0.02)
    assert np.array_equal(acc.cpu().numpy()[:, rows], acc_ref)
    assert np.array_equal(y.cpu().numpy()[:, rows].view(np.uint16), y_ref.view(np.uint16))


@pytest.mark.parametrize("M,K,N", SMALL_M_ONEBIT)
def test_onebit_prefill_small_token_counts(blw, oref, M, K, N):
    x, ws, g, h = _onebit_inputs(M, K, N, seed=4_100_000 + M + N)
    y = blw.ob_linear(x.cuda(), blw.ob_pack_sign(ws.cuda()), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    rows = _sample_rows(N, seed=M + 1)
    _, z_ref = oref.ob_linear(x.numpy(), oref.pack_sign(ws.numpy()[rows]), g.numpy(), h.numpy()[rows])
    assert _rel_err(y.cpu().numpy()[:, rows], z_ref) <= OB_TOL


def test_onebit_prefill_13b_full_size_sampled_rows(blw, oref):
    """The 13B-shaped down layer (K=13824, N=5120) at M=256, sampled rows."""
    M, K, N = 256, 13824, 5120
    assert blw.ob_workspace_bytes(M, K, N) >= 3 * M * K   # three limb planes
    x, ws, g, h = _onebit_inputs(M, K, N, seed=4_000_000)
    y = blw.ob_linear(x.cuda(), blw.ob_pack_sign(ws.cuda()), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    rows = np.sort(np.random.default_rng(6).choice(N, size=64, replace=False))
    s1s = oref.pack_sign(ws.numpy()[rows])
    _, z_ref = oref.ob_linear(x.numpy(), s1s, g.numpy(), h.numpy()[rows])
    assert _rel_err(y.cpu().numpy()[:, rows], z_ref) <= OB_TOL


def test_decode_full_size_layers(blw, oref):
    """Whole 7B down-projection (K=11008, N=4096) at M=1 and the 13B up layer
    (K=5120, N=13824) at M=4 against the oracle."""
    for (M, K, N, seed) in [(1, 11008, 4096, 91), (4, 5120, 13824, 92)]:
        x = synth.activations(M, K, seed=seed)
        w = synth.ternary_weights(N, K, seed=seed + 1)
        w2 = oref.pack_ternary(w.numpy())
        y, acc = blw.bl_ternary_linear(x.cuda(), torch.from_numpy(w2.view(np.int32)).cuda(), 0.02,
                                       return_acc=True)
        torch.cuda.synchronize()
        y_ref, acc_ref = oref.ternary_linear(x.numpy(), w2, 0.02)
        assert np.array_equal(acc.cpu().numpy(), acc_ref)


# ----------------------------------- fused decode chains and fallbacks -----

def test_fallback_two_kernel_path(blw, oref):
    """Shapes whose fused-decode shared memory would not fit take the
    activation-kernel + skinny-kernel path; both forms stay exact."""
    M, K, N = 8, 28672, 64
    x = synth.activations(M, K, seed=101)
    w2 = oref.pack_ternary(synth.ternary_weights(N, K, seed=102).numpy())
    y, acc = blw.bl_ternary_linear(x.cuda(), torch.from_numpy(w2.view(np.int32)).cuda(), 0.02,
                                   return_acc=True)
    torch.cuda.synchronize()
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), w2, 0.02)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    M, K, N = 16, 13824, 64
    x, ws, g, h = _onebit_inputs(M, K, N, seed=103)
    s1 = oref.pack_sign(ws.numpy())
    y = blw.ob_linear(x.cuda(), torch.from_numpy(s1.view(np.int32)).cuda(), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    _, z_ref = oref.ob_linear(x.numpy(), s1, g.numpy(), h.numpy())
    assert _rel_err(y.cpu().numpy(), z_ref) <= OB_TOL


@pytest.mark.parametrize("use_graph", [False, True])
def test_dependent_decode_chain(blw, oref, use_graph):
    """Eight M=1 layers where each layer's output is the next layer's input.
    The decode kernel streams weights before its programmatic-launch wait and
    reads x after it; the chained outputs must equal the oracle's chain
    bit for bit."""
    K = N = 1024
    layers = 8
    ws = [synth.ternary_weights(N, K, seed=200 + i) for i in range(layers)]
    w2s = [oref.pack_ternary(w.numpy()) for w in ws]
    w2d = [torch.from_numpy(w.view(np.int32)).cuda() for w in w2s]
    x0 = synth.activations(1, K, seed=199)
    xd = x0.cuda()
    bufs = [torch.empty((1, N), dtype=torch.float16, device="cuda") for _ in range(layers)]
    wsp = torch.empty((blw.bl_ternary_workspace_bytes(1, K, N),), dtype=torch.uint8, device="cuda")

    # keeps |y| ~ |x| through the chain: Var(sum q*t) ~ (2K/3) Var(q)
    w_scale = float(np.float32(1.0 / np.sqrt(2.0 * K / 3.0)))

    def run():
        cur = xd
        for i in range(layers):
            blw.bl_ternary_linear(cur, w2d[i], w_scale, workspace=wsp, out=bufs[i])
            cur = bufs[i]

    if use_graph:
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            run()
        torch.cuda.current_stream().wait_stream(s)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            run()
        for b in bufs:
            b.zero_()
        g.replay()
    else:
        run()
    torch.cuda.synchronize()
    cur = x0.numpy()
    for i in range(layers):
        y_ref, _ = oref.ternary_linear(cur, w2s[i], w_scale)
        assert np.all(np.isfinite(y_ref.astype(np.float32)))
        assert np.array_equal(bufs[i].cpu().numpy().view(np.uint16), y_ref.view(np.uint16)), i
        cur = y_ref


def test_decode_all_token_counts_fused(blw, oref):
    """Every M the fused decode kernel serves (ternary 1..32), one shape each."""
    K, N = 640, 48
    w = synth.ternary_weights(N, K, seed=300)
    w2 = oref.pack_ternary(w.numpy())
    w2d = torch.from_numpy(w2.view(np.int32)).cuda()
    for M in range(1, 33):
        x = synth.activations(M, K, seed=300 + M)
        y, acc = blw.bl_ternary_linear(x.cuda(), w2d, 0.02, return_acc=True)
        torch.cuda.synchronize()
        _, acc_ref = oref.ternary_linear(x.numpy(), w2, 0.02)
        assert np.array_equal(acc.cpu().numpy(), acc_ref), M


@pytest.mark.parametrize("M,K,N", [(2, 4096, 272), (3, 4096, 272), (5, 4096, 48), (8, 4096, 4096),
                                   (4, 2048, 64), (8, 1024, 96), (2, 11008, 64)])
def test_decode_warp_local_multi_token(blw, oref, M, K, N):
    """Small-M calls whose activations each warp prepares for exactly the
    k-steps it contracts (up to four token/group units per lane; K = 2048 and
    1024 leave warps that own no step)."""
    x = synth.activations(M, K, seed=400 + M + K, outlier_frac=0.01)
    w2 = oref.pack_ternary(synth.ternary_weights(N, K, seed=401 + M).numpy())
    y, acc = blw.bl_ternary_linear(x.cuda(), torch.from_numpy(w2.view(np.int32)).cuda(), 0.02,
                                   return_acc=True)
    torch.cuda.synchronize()
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), w2, 0.02)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    assert np.array_equal(y.cpu().numpy().view(np.uint16), y_ref.view(np.uint16))


@pytest.mark.parametrize("M,K,N", [(2, 4096, 48), (2, 384, 32), (1, 8192, 64), (2, 11008, 32)])
def test_onebit_decode_warp_local_two_tokens(blw, oref, M, K, N):
    """OneBit at M <= 2 with warp-local preparation (partial last step for
    K = 384 and 11008)."""
    x, ws, g, h = _onebit_inputs(M, K, N, seed=420 + M + K)
    s1 = oref.pack_sign(ws.numpy())
    y = blw.ob_linear(x.cuda(), torch.from_numpy(s1.view(np.int32)).cuda(), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    _, z_ref = oref.ob_linear(x.numpy(), s1, g.numpy(), h.numpy())
    assert _rel_err(y.cpu().numpy(), z_ref) <= OB_TOL


@pytest.mark.parametrize("M", [1, 4, 12, 20])
def test_quant_two_step_rounding_on_every_path(blw, oref, M):
    """x = amax/2 whose fp32 product with rn(127/amax) is exactly 63.5 (the exact
    product is just below it): every activation path must round the fp32 product,
    giving 64, like the oracle (M = 1 and 4: in-kernel warp-local preparation;
    12: the activation kernel; 20: the activation kernel before the tensor-core GEMM)."""
    K, N = 4096, 64
    x = synth.activations(M, K, seed=500 + M)
    amax = np.float16(4.6328125)
    x[:, :] = torch.clamp(x, -4.5, 4.5)
    x[:, 7] = float(amax)
    x[:, 100] = float(np.float16(amax / 2))
    x[:, 2049] = -float(np.float16(amax / 2))
    w2 = oref.pack_ternary(synth.ternary_weights(N, K, seed=501).numpy())
    y, acc = blw.bl_ternary_linear(x.cuda(), torch.from_numpy(w2.view(np.int32)).cuda(), 0.02,
                                   return_acc=True)
    torch.cuda.synchronize()
    q_ref, _ = oref.quant_act(x.numpy())
    assert q_ref[0, 100] == 64 and q_ref[0, 2049] == -64
    _, acc_ref = oref.ternary_linear(x.numpy(), w2, 0.02)
    assert np.array_equal(acc.cpu().numpy(), acc_ref)
    q, s = blw.bl_quant_act(x.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)


# ------------------------------------- OneBit tokens dominated by one value --

def _per_token_rel_err(y, z_ref):
    """max over tokens of max_n |y - z_ref| / max_n |z_ref| (each token against
    its own scale: stricter than one max over the whole output)."""
    y = np.asarray(y, dtype=np.float64)
    den = np.max(np.abs(z_ref), axis=1)
    den[den == 0] = 1.0
    return float(np.max(np.max(np.abs(y - z_ref), axis=1) / den))


# (M, K, N) reaching every OneBit path: M = 1 and 2 prepare the activations in
# the streamed decode kernel (warp-local), M = 4 through the activation kernel
# and the prepared streamed kernel, M = 16 the small-token tensor-core tiles,
# M = 256 the full tensor-core tiles; K = 65536 (M = 1, 4) takes the two-pass
# activation kernel and the skinny fallback.
OUTLIER_SHAPES = [(M, K, N) for (K, N) in [(4096, 4096), (13824, 5120)] for M in (1, 2, 4, 16, 256)]
OUTLIER_SHAPES += [(1, 65536, 32), (4, 65536, 32)]


@pytest.mark.parametrize("val", [2000.0, -60000.0])
@pytest.mark.parametrize("M,K,N", OUTLIER_SHAPES)
def test_onebit_outlier_tokens_every_path(blw, oref, M, K, N, val):
    """A token holding one activation of 2000 or -60000 among N(0,1) values:
    that element sets the token's fixed-point step, so the rest of the token
    is resolved at step = max|x*g| / (2^22 - 1).  Every token must stay within
    2e-3 of its own largest output."""
    x, ws, g, h = _onebit_inputs(M, K, N, seed=4_200_000 + M + K + int(val))
    x[0, 17] = val
    if M > 1:
        x[M - 1, K - 3] = -val
        x[M // 2, K // 2 + 1] = val / 3
    y = blw.ob_linear(x.cuda(), blw.ob_pack_sign(ws.cuda()), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    rows = np.arange(N)
    if M * N * K > 2e8:   # 128 sampled rows, first and last included
        rows = np.sort(np.random.default_rng(M + 3).choice(N, size=128, replace=False))
        rows[0], rows[-1] = 0, N - 1
    _, z_ref = oref.ob_linear(x.numpy(), oref.pack_sign(ws.numpy()[rows]), g.numpy(), h.numpy()[rows])
    assert _per_token_rel_err(y.cpu().numpy()[:, rows], z_ref) <= OB_TOL


# ------------------------------------------- largest sweep and 70B shapes ----

@pytest.mark.parametrize("K,N", [(5120, 13824), (13824, 5120)])
def test_ternary_m1024_13b_sampled_rows(blw, oref, K, N):
    """The batch sweep's largest token count (M = 1024) on both 13B-shaped
    layers: int32 accumulators and y bit-exact on sampled rows (first and last
    included)."""
    M = 1024
    x = synth.activations(M, K, seed=4_300_000 + K, outlier_frac=0.01)
    w = synth.ternary_weights(N, K, seed=4_300_001 + K)
    y, acc = blw.bl_ternary_linear(x.cuda(), blw.bl_pack_ternary(w.cuda()), 0.02, return_acc=True)
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    rows = _sample_rows(N, seed=11)
    y_ref, acc_ref = oref.ternary_linear(x.numpy(), oref.pack_ternary(w.numpy()[rows]), 0.02)
    assert np.array_equal(acc.cpu().numpy()[:, rows], acc_ref)
    assert np.array_equal(y.cpu().numpy()[:, rows].view(np.uint16), y_ref.view(np.uint16))


@pytest.mark.parametrize("M,K,N", [(1024, 5120, 13824), (1024, 13824, 5120), (512, 8192, 28672)])
def test_onebit_large_m_sampled_rows(blw, oref, M, K, N):
    """OneBit at the batch sweep's M = 1024 on both 13B-shaped layers and at
    M = 512 on the 70B-shaped 8192->28672 layer, sampled rows."""
    x, ws, g, h = _onebit_inputs(M, K, N, seed=4_400_000 + M + K)
    y = blw.ob_linear(x.cuda(), blw.ob_pack_sign(ws.cuda()), g.cuda(), h.cuda())
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    rows = _sample_rows(N, seed=13)
    _, z_ref = oref.ob_linear(x.numpy(), oref.pack_sign(ws.numpy()[rows]), g.numpy(), h.numpy()[rows])
    assert _per_token_rel_err(y.cpu().numpy()[:, rows], z_ref) <= OB_TOL
