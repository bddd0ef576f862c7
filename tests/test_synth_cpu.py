"""The seeded input generators produce the input recipe of the tests and the benchmark -- latent
weights N(0, 0.02^2), activations N(0, 1), forget pre-activations N(4, 1) (long memory) or N(0, 1),
input pre-activations N(0, 1), token ids uniform in [0, 32000), gains ones or N(1, 0.1^2), the model
table's shapes -- reproducibly from their seeds, and hold none of the method's arithmetic."""
import numpy as np
import pytest

import synth


def test_draws_are_seeded_and_reproducible():
    assert np.array_equal(synth.activations(5, (3, 4)), synth.activations(5, (3, 4)))
    assert not np.array_equal(synth.activations(5, (3, 4)), synth.activations(6, (3, 4)))
    a, b = synth.scan_inputs(7, 2, 3, 4, True), synth.scan_inputs(7, 2, 3, 4, True)
    assert all(np.array_equal(x, y) for x, y in zip(a, b))


def test_distributions_of_the_recipe():
    w = synth.weight(1, 1000, 1000)
    assert w.dtype == np.float32 and w.shape == (1000, 1000)
    assert abs(float(w.mean())) < 1e-4 and abs(float(w.std()) - 0.02) < 2e-4          # N(0, 0.02^2)
    x = synth.activations(2, (1000, 1000))
    assert abs(float(x.mean())) < 5e-3 and abs(float(x.std()) - 1.0) < 5e-3           # N(0, 1)
    zf, zi = synth.scan_inputs(3, 4, 256, 256, long_memory=True)
    assert abs(float(zf.mean()) - 4.0) < 1e-2 and abs(float(zf.std()) - 1.0) < 1e-2   # N(4, 1)
    assert abs(float(zi.mean())) < 1e-2 and abs(float(zi.std()) - 1.0) < 1e-2
    zf0, _ = synth.scan_inputs(3, 4, 256, 256, long_memory=False)
    assert abs(float(zf0.mean())) < 1e-2                                                  # N(0, 1)
    ids = synth.token_ids(4, (200000,))
    assert ids.dtype == np.int32 and ids.min() >= 0 and ids.max() < synth.VOCAB
    assert abs(float(ids.mean()) - (synth.VOCAB - 1) / 2) < 0.01 * synth.VOCAB          # uniform
    assert np.all(synth.norm_weight(5, 64) == 1.0)
    g = synth.norm_weight(5, 100000, random=True)
    assert abs(float(g.mean()) - 1.0) < 2e-3 and abs(float(g.std()) - 0.1) < 2e-3      # N(1, 0.1^2)
    e = synth.embedding(6, 32000, 64)
    assert e.shape == (32000, 64) and abs(float(e.std()) - 0.02) < 2e-4


@pytest.mark.parametrize("shape", [synth.TINY, synth.M370, synth.B13, synth.B27], ids=lambda s: s.name)
def test_block_params_follow_the_model_table(shape):
    if shape.d > 1024:                       # the large shapes: sizes only (no draw)
        ps = shape.proj_shapes
        assert ps["gate"] == (2 * shape.inner, shape.d) and ps["down"] == (shape.d, shape.inner)
        return
    p = synth.block_params(9, shape, random_norms=True)
    for name, (n, k) in shape.proj_shapes.items():
        assert p[f"W_{name}"].shape == (n, k) and p[f"W_{name}"].dtype == np.float32
        assert p[f"nw_{name}"].shape == (k,)
    assert p["gnorm_w"].shape == (shape.d,)
    # distinct projections get distinct draws
    assert not np.array_equal(p["W_i"], p["W_f"])


def test_generators_hold_no_arithmetic_of_the_method():
    import inspect

    src = inspect.getsource(synth)
    for word in ("rint", "round(", "sigmoid", "exp(", "sqrt", "clip(", "cumprod", "tanh"):
        assert word not in src, word
