"""The seeded input generators (shared by the oracle tests and the CUDA path)
are reproducible and draw the stated distributions; they hold none of the
layer's arithmetic."""
import torch

from bit_weight_linear_b200 import synth


def test_generators_are_reproducible_and_seed_dependent():
    for f, args in [(synth.activations, (3, 256)), (synth.ternary_weights, (16, 256)),
                    (synth.sign_weights, (16, 256)), (synth.value_vector, (256,)),
                    (synth.norm_weight, (256,)), (synth.svid_weights, (16, 256))]:
        a, b, c = f(*args, seed=5), f(*args, seed=5), f(*args, seed=6)
        assert torch.equal(a, b), f.__name__
        assert not torch.equal(a, c), f.__name__


def test_distributions():
    t = synth.ternary_weights(256, 1024, seed=1)
    assert set(t.unique().tolist()) == {-1, 0, 1}
    assert abs((t == 0).float().mean().item() - 1 / 3) < 0.01
    s = synth.sign_weights(256, 1024, seed=2)
    assert set(s.unique().tolist()) == {-1.0, 1.0}
    g = synth.value_vector(4096, seed=3).float()
    assert 0.01 - 1e-4 <= g.min().item() and g.max().item() <= 0.03 + 1e-4
    n = synth.norm_weight(4096, seed=4).float()
    assert abs(n.mean().item() - 1.0) < 0.01 and abs(n.std().item() - 0.1) < 0.01
    x = synth.activations(1, 10000, seed=5, outlier_frac=0.01, outlier_mult=20.0).float()[0]
    assert (x.abs() > 10).sum().item() >= 50          # about 100 channels scaled x20
    w = synth.svid_weights(256, 256, seed=6)
    assert w.dtype == torch.float32 and abs(w.std().item() - 0.02) < 0.002
