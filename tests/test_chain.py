"""Decode chains: the single-token forward of a list of layers in one
persistent launch (bl_chain_build / bl_chain_run), against the oracle.

Each layer is checked on its own: the oracle is applied to the input the GPU
layer actually read (the given x, or the GPU's output of the producing layer),
so a layer's check does not depend on the others.  Ternary layers must match
bit for bit (int32 accumulators and fp16 outputs); OneBit layers within 2e-3
of the token's largest output."""
import numpy as np
import pytest
import torch

from bit_weight_linear_b200 import synth

pytestmark = pytest.mark.gpu

OB_TOL = 2e-3
BLOCK_7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
            ("gate", 4096, 11008), ("up", 4096, 11008), ("down", 11008, 4096)]


@pytest.fixture(scope="module")
def blw():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_weight_linear_b200 import build
    build.build()
    import bit_weight_linear_b200 as m
    return m


def block_sources(blocks):
    """The dependency pattern of a LLaMA-like decode step through the 7-layer
    block, with each elementwise step between two linears replaced by the
    identity: q, k, v read the block input (block 0: a given x; later blocks:
    the previous block's down output), o reads v's output (attention's place),
    gate and up read o's output (the residual/norm's place), down reads gate's
    output (SwiGLU's place)."""
    src = []
    for b in range(blocks):
        base = 7 * b
        blk_in = -1 if b == 0 else base - 1
        src += [blk_in, blk_in, blk_in, base + 2, base + 3, base + 3, base + 4]
    return src


def ternary_chain(blw, shapes, srcs, seed, acc=True):
    layers, host = [], []
    x0 = None
    for j, ((K, N), s) in enumerate(zip(shapes, srcs)):
        w = synth.ternary_weights(N, K, seed=seed + 3 * j)
        d = dict(K=K, N=N, w=blw.bl_pack_ternary(w.cuda()),
                 # keeps |y| ~ |x| along the chain: Var(sum q t) ~ (2K/3) Var(q)
                 w_scale=float(np.float32(1.0 / np.sqrt(2.0 * K / 3.0))),
                 y=torch.empty((N,), dtype=torch.float16, device="cuda"), src=s)
        if acc:
            d["acc_out"] = torch.empty((N,), dtype=torch.int32, device="cuda")
        if s < 0:
            x = synth.activations(1, K, seed=seed + 3 * j + 1, outlier_frac=0.01)[0]
            d["x"] = x.cuda()
        layers.append(d)
        host.append(w)
    return layers, host


def check_ternary(oref, layers, host):
    for j, (d, w) in enumerate(zip(layers, host)):
        xin = d["x"] if d["src"] < 0 else layers[d["src"]]["y"]
        y_ref, acc_ref = oref.ternary_linear(xin.cpu().numpy()[None, :], oref.pack_ternary(w.numpy()),
                                             d["w_scale"], parallel=True)
        if "acc_out" in d:
            assert np.array_equal(d["acc_out"].cpu().numpy(), acc_ref[0]), j
        assert np.array_equal(d["y"].cpu().numpy().view(np.uint16), y_ref[0].view(np.uint16)), j


def test_chain_llama7b_stack_32_blocks_dependent_bit_exact(blw, oref):
    """The whole LLaMA-7B-shaped decode stack (32 blocks x 7 layers) in one
    launch, with the dependency pattern of a decode step; run twice (the
    completion counters restart at zero every run)."""
    blocks = 32
    shapes = [(K, N) for _ in range(blocks) for (_, K, N) in BLOCK_7B]
    layers, host = ternary_chain(blw, shapes, block_sources(blocks), seed=600_000, acc=False)
    ch = blw.Chain(0, layers)
    for _ in range(2):
        for d in layers:
            d["y"].zero_()
        ch.run()
        torch.cuda.synchronize()
        assert blw.bl_device_status() == 0
    # every layer's y is finite (the chain keeps |y| ~ 1) and exact
    assert all(torch.isfinite(d["y"].float()).all() for d in layers)
    check_ternary(oref, layers, host)


# (K, N) edge shapes: one tile (most CTAs idle), a ragged last step (640 ->
# 160 packed bytes per row), 43-step rows in three stages (11008), 13 tiles per
# CTA (28672), the 70B down layer (K = 28672), and two layers sharing an input
INDEPENDENT = [(4096, 16), (640, 48), (11008, 4096), (4096, 28672), (28672, 256), (1024, 1024),
               (1024, 512)]


def test_chain_independent_edge_shapes(blw, oref):
    layers, host = ternary_chain(blw, INDEPENDENT, [-1] * len(INDEPENDENT), seed=610_000)
    layers[-1]["x"] = layers[-2]["x"]       # same input as the layer before: reused activations
    ch = blw.Chain(0, layers)
    ch.run()
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    check_ternary(oref, layers, host)


def test_chain_matches_per_call_entry_point(blw):
    """A chain of independent layers gives exactly what one bl_ternary_linear
    call per layer gives."""
    shapes = [(4096, 4096), (4096, 11008), (11008, 4096)]
    layers, _ = ternary_chain(blw, shapes, [-1, -1, -1], seed=620_000)
    blw.Chain(0, layers).run()
    for d in layers:
        y, acc = blw.bl_ternary_linear(d["x"][None, :], d["w"], d["w_scale"], return_acc=True)
        torch.cuda.synchronize()
        assert torch.equal(acc[0], d["acc_out"])
        assert torch.equal(y[0].view(torch.int16), d["y"].view(torch.int16))


def _onebit_chain(blw, shapes, srcs, seed):
    layers, host = [], []
    for j, ((K, N), s) in enumerate(zip(shapes, srcs)):
        w = synth.sign_weights(N, K, seed=seed + 5 * j)
        # value vectors scaled so that |y| ~ |x| along the chain
        g = (synth.value_vector(K, seed=seed + 5 * j + 1).float() * (50.0 / np.sqrt(K))).half()
        h = (synth.value_vector(N, seed=seed + 5 * j + 2).float() * 50.0).half()
        d = dict(K=K, N=N, w=blw.ob_pack_sign(w.cuda()), g=g.cuda(), h=h.cuda(), src=s,
                 y=torch.empty((N,), dtype=torch.float16, device="cuda"))
        if s < 0:
            x = synth.activations(1, K, seed=seed + 5 * j + 3)[0]
            x[17] = 2000.0 if j % 2 == 0 else -60000.0     # one dominant activation
            d["x"] = x.cuda()
        layers.append(d)
        host.append((w, g, h))
    return layers, host


def test_chain_onebit_dependent_and_edge_shapes(blw, oref):
    shapes = [(4096, 4096), (4096, 4096), (4096, 11008), (11008, 4096), (384, 48), (13824, 5120),
              (5120, 16)]
    srcs = [-1, 0, 1, 2, -1, -1, 5]
    layers, host = _onebit_chain(blw, shapes, srcs, seed=630_000)
    blw.Chain(1, layers).run()
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    for j, (d, (w, g, h)) in enumerate(zip(layers, host)):
        xin = d["x"] if d["src"] < 0 else layers[d["src"]]["y"]
        _, z_ref = oref.ob_linear(xin.cpu().numpy()[None, :], oref.pack_sign(w.numpy()), g.numpy(),
                                  h.numpy(), parallel=True)
        y = d["y"].cpu().numpy().astype(np.float64)
        assert np.max(np.abs(y - z_ref[0])) <= OB_TOL * np.max(np.abs(z_ref[0])), j


def fused_block_layers(blocks):
    """The LLaMA-like decode step with its fused steps: q, k, v read
    RMSNorm(block input); o reads v's output (attention's place, identity);
    gate and up read RMSNorm(o's output); down reads SwiGLU(gate, up).
    Returns (src, src2, has_norm) per layer."""
    out = []
    for b in range(blocks):
        base = 7 * b
        blk_in = -1 if b == 0 else base - 1
        out += [(blk_in, -1, True), (blk_in, -1, True), (blk_in, -1, True), (base + 2, -1, False),
                (base + 3, -1, True), (base + 3, -1, True), (base + 4, base + 5, False)]
    return out


def _fused_input(oref, layers, d):
    """The fp16 input a fused layer quantises, from the oracle's RMSNorm and
    SwiGLU applied to what the GPU layer read."""
    xin = (d["x"] if d["src"] < 0 else layers[d["src"]]["y"]).cpu().numpy()
    if d.get("src2", -1) >= 0:
        xin = oref.swiglu(xin, layers[d["src2"]]["y"].cpu().numpy())
    if d.get("norm_w") is not None:
        xin = oref.rmsnorm(xin[None, :], d["norm_w"].cpu().numpy(), d["norm_eps"])[0]
    return xin


EPS = float(np.float32(1e-5))


def test_chain_fused_llama7b_blocks_bit_exact(blw, oref):
    """Four LLaMA-7B blocks with RMSNorm and SwiGLU fused into the chain: every
    layer's accumulators and outputs equal the oracle's RMSNorm / SwiGLU /
    BitLinear applied to the GPU's own inputs, bit for bit.  Blocks 0 and 2
    evaluate SwiGLU once per element in up's epilogue (swiglu_buf, checked
    against the oracle's SwiGLU too); blocks 1 and 3 in every CTA."""
    blocks = 4
    shapes = [(K, N) for _ in range(blocks) for (_, K, N) in BLOCK_7B]
    plan = fused_block_layers(blocks)
    layers, host = ternary_chain(blw, shapes, [s for s, _, _ in plan], seed=640_000)
    for j, (d, (_, s2, norm)) in enumerate(zip(layers, plan)):
        d["src2"] = s2
        if s2 >= 0 and (j // 7) % 2 == 0:
            d["swiglu_buf"] = torch.full((d["K"],), float("nan"), dtype=torch.float16, device="cuda")
        if norm:
            # q, k, v (and gate, up) share one RMSNorm weight: prepared once
            d["norm_w"] = synth.norm_weight(d["K"], seed=641_000 + (j // 7) * 2 + (j % 7 >= 4)).cuda()
            d["norm_eps"] = EPS
    for j in range(1, len(layers)):
        if plan[j][2] and plan[j - 1][2] and plan[j][0] == plan[j - 1][0]:
            layers[j]["norm_w"] = layers[j - 1]["norm_w"]
    ch = blw.Chain(0, layers)
    for _ in range(2):
        for d in layers:
            d["y"].zero_()
        ch.run()
        torch.cuda.synchronize()
        assert blw.bl_device_status() == 0
    for j, (d, w) in enumerate(zip(layers, host)):
        xin = _fused_input(oref, layers, d)
        assert np.isfinite(xin.astype(np.float32)).all(), j
        if "swiglu_buf" in d:
            assert np.array_equal(d["swiglu_buf"].cpu().numpy().view(np.uint16), xin.view(np.uint16)), j
        y_ref, acc_ref = oref.ternary_linear(xin[None, :], oref.pack_ternary(w.numpy()), d["w_scale"],
                                             parallel=True)
        assert np.array_equal(d["acc_out"].cpu().numpy(), acc_ref[0]), j
        assert np.array_equal(d["y"].cpu().numpy().view(np.uint16), y_ref[0].view(np.uint16)), j


def test_chain_fused_prologue_edge_rows(blw, oref):
    """RMSNorm at the largest fused row (17920) and on a zero row (r =
    1/sqrt(eps)); SwiGLU of a row whose gate values reach +-5e3 (exp(-a)
    overflows to inf: silu -> -0) and of two rows in either order."""
    K1 = 17920
    shapes = [(K1, 256), (1024, 128), (1024, 1024), (128, 1024), (1024, 64), (1024, 64)]
    layers, host = ternary_chain(blw, shapes, [-1, -1, -1, -1, 2, 3], seed=650_000)
    layers[0]["norm_w"], layers[0]["norm_eps"] = synth.norm_weight(K1, seed=650_100).cuda(), EPS
    layers[1]["x"].zero_()
    layers[1]["norm_w"], layers[1]["norm_eps"] = synth.norm_weight(1024, seed=650_101).cuda(), 0.25
    # y2 large (|y2| ~ 2e3, beyond exp overflow at 709) but silu(y2) * y3 finite
    x2 = layers[2]["x"].float()
    x2[::7] = 60000.0
    x2[1::7] = -60000.0
    layers[2]["x"].copy_(x2.half())
    layers[2]["w_scale"] = 0.002
    layers[4]["src2"] = 3                   # SwiGLU(y2, y3), evaluated in layer 3's epilogue
    layers[5]["src2"] = 2                   # SwiGLU(y3, y2), then RMSNorm: layer 3 already
    for d in layers[4:]:                    # evaluates the other order, so every CTA does this one
        d["swiglu_buf"] = torch.empty((1024,), dtype=torch.float16, device="cuda")
    layers[5]["norm_w"], layers[5]["norm_eps"] = synth.norm_weight(1024, seed=650_102).cuda(), EPS
    blw.Chain(0, layers).run()
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    y2 = layers[2]["y"].float()
    assert torch.isfinite(y2).all() and y2.abs().max() > 1000.0
    for j, (d, w) in enumerate(zip(layers, host)):
        xin = _fused_input(oref, layers, d)
        assert np.isfinite(xin.astype(np.float32)).all(), j
        y_ref, acc_ref = oref.ternary_linear(xin[None, :], oref.pack_ternary(w.numpy()), d["w_scale"],
                                             parallel=True)
        assert np.array_equal(d["acc_out"].cpu().numpy(), acc_ref[0]), j
        assert np.array_equal(d["y"].cpu().numpy().view(np.uint16), y_ref[0].view(np.uint16)), j


def test_chain_fused_onebit_block(blw, oref):
    """The fused block on OneBit layers (row widths up to 11008 < 14336)."""
    shapes = [(K, N) for (_, K, N) in BLOCK_7B]
    plan = fused_block_layers(1)
    layers, host = _onebit_chain(blw, shapes, [s for s, _, _ in plan], seed=660_000)
    nw = [synth.norm_weight(4096, seed=660_100 + i).cuda() for i in range(2)]
    for j, (d, (_, s2, norm)) in enumerate(zip(layers, plan)):
        d["src2"] = s2
        if s2 >= 0:
            d["swiglu_buf"] = torch.empty((d["K"],), dtype=torch.float16, device="cuda")
        if norm:
            d["norm_w"], d["norm_eps"] = nw[j >= 4], EPS
    blw.Chain(1, layers).run()
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    for j, (d, (w, g, h)) in enumerate(zip(layers, host)):
        xin = _fused_input(oref, layers, d)
        _, z_ref = oref.ob_linear(xin[None, :], oref.pack_sign(w.numpy()), g.numpy(), h.numpy(),
                                  parallel=True)
        y = d["y"].cpu().numpy().astype(np.float64)
        assert np.max(np.abs(y - z_ref[0])) <= OB_TOL * np.max(np.abs(z_ref[0])), j


def test_chain_swiglu_buffer_either_order(blw, oref):
    """SwiGLU evaluated once per element in the producing epilogue, with the
    gate as the later layer (SwiGLU(y_later, y_earlier)) and as the earlier
    one, on OneBit-free ternary layers of different widths; the buffers hold
    exactly the oracle's SwiGLU of the GPU's outputs."""
    shapes = [(512, 1536), (512, 1536), (1536, 256), (1536, 256)]
    layers, host = ternary_chain(blw, shapes, [-1, -1, 1, 0], seed=670_000)
    layers[2]["src2"] = 0          # SwiGLU(y1, y0): the producer (layer 1) is the gate
    layers[3]["src2"] = 1          # SwiGLU(y0, y1): layer 1 already evaluates the other order
    for d in layers[2:]:
        d["swiglu_buf"] = torch.full((1536,), float("nan"), dtype=torch.float16, device="cuda")
    blw.Chain(0, layers).run()
    torch.cuda.synchronize()
    assert blw.bl_device_status() == 0
    h = oref.swiglu(layers[1]["y"].cpu().numpy(), layers[0]["y"].cpu().numpy())
    assert np.array_equal(layers[2]["swiglu_buf"].cpu().numpy().view(np.uint16), h.view(np.uint16))
    for j, (d, w) in enumerate(zip(layers, host)):
        xin = _fused_input(oref, layers, d)
        y_ref, acc_ref = oref.ternary_linear(xin[None, :], oref.pack_ternary(w.numpy()), d["w_scale"])
        assert np.array_equal(d["acc_out"].cpu().numpy(), acc_ref[0]), j
        assert np.array_equal(d["y"].cpu().numpy().view(np.uint16), y_ref[0].view(np.uint16)), j


def test_chain_run_host_matches_device_run(blw):
    """bl_chain_run_host: the given input copied from pinned host memory, the
    chain, every output copied back, on one stream; identical to run() on the
    same input."""
    shapes = [(1024, 512), (512, 256)]
    layers, _ = ternary_chain(blw, shapes, [-1, 0], seed=680_000)
    ch = blw.Chain(0, layers)
    ch.run()
    torch.cuda.synchronize()
    ref = [d["y"].cpu() for d in layers]
    xin = layers[0]["x"].cpu().pin_memory()
    layers[0]["x"].zero_()
    outs = [torch.zeros(d["y"].shape, dtype=torch.float16).pin_memory() for d in layers]
    for d in layers:
        d["y"].zero_()
    ch.run_host([(xin, layers[0]["x"])], [(d["y"], o) for d, o in zip(layers, outs)])
    torch.cuda.current_stream().synchronize()
    assert blw.bl_device_status() == 0
    for o, r in zip(outs, ref):
        assert torch.equal(o.view(torch.int16), r.view(torch.int16))
