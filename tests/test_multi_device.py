"""Every launch path on two devices from one process: the kernel attributes
(dynamic shared memory, carveout) are set per device, so a call on the second
device after calls on the first must work and give the same results.  Skipped
unless two CUDA devices are visible."""
import pytest
import torch

from bit_weight_linear_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def blw():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    if torch.cuda.device_count() < 2:
        pytest.skip("needs two visible CUDA devices")
    from bit_weight_linear_b200 import build
    build.build()
    import bit_weight_linear_b200 as m
    return m


def _run_all(blw, dev):
    out = {}
    with torch.cuda.device(dev):
        w = synth.ternary_weights(1024, 2048, seed=1).to(dev)
        w2 = blw.bl_pack_ternary(w)
        for M in (1, 4, 64):                       # streamed, prepared streamed, tensor-core
            x = synth.activations(M, 2048, seed=2 + M).to(dev)
            out[f"t{M}"] = blw.bl_ternary_linear(x, w2, 0.02)
        s = synth.sign_weights(1024, 2048, seed=3).to(dev)
        s1 = blw.ob_pack_sign(s)
        g = synth.value_vector(2048, seed=4).to(dev)
        h = synth.value_vector(1024, seed=5).to(dev)
        for M in (1, 3, 16):
            x = synth.activations(M, 2048, seed=6 + M).to(dev)
            out[f"o{M}"] = blw.ob_linear(x, s1, g, h)
        layers = [dict(K=2048, N=1024, x=synth.activations(1, 2048, seed=9)[0].to(dev), w=w2,
                       w_scale=0.02, y=torch.empty((1024,), dtype=torch.float16, device=dev)),
                  dict(K=1024, N=1024, src=0, w=blw.bl_pack_ternary(synth.ternary_weights(1024, 1024, seed=10).to(dev)),
                       w_scale=0.03, y=torch.empty((1024,), dtype=torch.float16, device=dev))]
        blw.Chain(0, layers).run()
        out["chain"] = layers[1]["y"]
        W = synth.svid_weights(256, 512, seed=11).to(dev)
        out["svid_h"] = blw.ob_svid(W)[2]
        b2, alpha = blw.billm_binarize(W)
        out["billm"] = blw.billm_linear(synth.activations(2, 512, seed=12).to(dev), b2, alpha)
        torch.cuda.synchronize(dev)
        assert blw.bl_device_status() == 0
    return {k: v.cpu() for k, v in out.items()}


def test_every_path_on_two_devices(blw):
    a = _run_all(blw, 0)
    b = _run_all(blw, 1)
    for k in a:
        assert torch.equal(a[k].view(torch.int16), b[k].view(torch.int16)), k
