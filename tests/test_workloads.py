"""The seeded input generator: determinism, block independence, ranges."""
import numpy as np
import pytest

from kalman_linear_attention_b200 import workloads as wl


def test_block_size_does_not_change_values():
    w = wl.WORKLOADS["tiny"].with_shape(B=3, T=37, H=2, N=5)
    full = wl.generate(w)
    for rows in (1, 7, 1000):
        got = {k: [] for k in wl.INPUT_NAMES}
        for r0, r1, blk in wl.iter_rows(w, rows_per_block=rows):
            for k in wl.INPUT_NAMES:
                got[k].append(blk[k])
        for k in wl.INPUT_NAMES:
            np.testing.assert_array_equal(np.concatenate(got[k]).reshape(full[k].shape), full[k])


def test_deterministic_and_seed_dependent():
    w = wl.WORKLOADS["stiff"].with_shape(B=2, T=8)
    x1, x2 = wl.generate(w), wl.generate(w)
    x3 = wl.generate(w.with_shape(seed=w.seed + 1))
    for k in wl.INPUT_NAMES:
        np.testing.assert_array_equal(x1[k], x2[k])
        assert not np.array_equal(x1[k], x3[k])


@pytest.mark.parametrize("name", ["tiny", "lm_layer", "stiff"])
def test_ranges(name):
    w = wl.WORKLOADS[name].with_shape(B=2, T=256, H=2, N=16)
    x = wl.generate(w)
    lo_hi = {"tiny": {"a": (0.5, 1.0), "p": (1e-3, 1.0), "phi": (1e-2, 10.0)},
             "stiff": {"a": (0.99, 1.0), "p": (1e-6, 1e-3), "phi": (1e-3, 1e3)},
             "lm_layer": {"a": (0.0, 1.0), "p": (0.0, 10.0), "phi": (0.0, 20.0)}}[name]
    for k, (lo, hi) in lo_hi.items():
        assert x[k].min() >= lo * (1 - 1e-6) and x[k].max() <= hi * (1 + 1e-6), k
    assert abs(x["b"].mean()) < 0.05 and abs(x["b"].std() - 1) < 0.05
    assert (x["lam0"] == 1).all() and (x["eta0"] == 0).all()


def test_bf16_values_are_representable():
    w = wl.WORKLOADS["lm_layer"].with_shape(B=1, T=64, H=2, N=8)
    x = wl.generate(w)
    for k in wl.INPUT_NAMES:
        bits = x[k].view(np.uint32)
        assert (bits & 0xFFFF == 0).all(), k


def test_bf16_rounding_ties_to_even():
    vals = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9], dtype=np.float32)
    got = wl.round_to_bf16(vals)
    np.testing.assert_array_equal(got, np.array([1.0, 1.0 + 2 ** -6, 1.0], dtype=np.float32))


def test_layer_generator_shapes_and_ranges():
    import dataclasses
    w = wl.LAYER_WORKLOADS["layer"].with_shape(B=2, T=40, H=2, D=6, Ns=8)
    x = wl.generate_layer(w)
    assert x["k"].shape == (2, 40, 2, 8) and x["v"].shape == (2, 40, 2, 6) and x["a"].shape == (2, 6, 8)
    assert np.all(x["w"] > 0) and np.all((x["a"] > 0) & (x["a"] < 1)) and np.all(x["p"] > 0)
    # bf16 workloads carry bf16-representable values
    assert np.array_equal(wl.round_to_bf16(x["k"]), x["k"])
    y = wl.generate_layer(w)
    assert all(np.array_equal(x[k], y[k]) for k in x)                    # seeded
    f32 = wl.generate_layer(dataclasses.replace(w, dtype="f32"))
    assert not np.array_equal(wl.round_to_bf16(f32["v"]), f32["v"])      # fp32 keeps its bits
    pr = wl.random_layer_prior(w)
    assert pr["lam0"].shape == (2, 2, 6, 8) and np.all(pr["lam0"] > 0)


def test_output_gradients_do_not_depend_on_block_size():
    w = wl.WORKLOADS["tiny"].with_shape(B=2, T=30, H=1, N=8)
    full = wl.generate_output_grads(w)
    parts = list(wl.iter_output_grad_rows(w, rows_per_block=7))
    for k in wl.GRAD_NAMES:
        cat = np.concatenate([blk[k] for _, _, blk in parts]).reshape(full[k].shape)
        assert np.array_equal(cat, full[k]), k


@pytest.mark.parametrize("kind", wl.SPECIAL_CASES)
def test_special_inputs(kind):
    x = wl.special_inputs(kind, T=50)
    assert np.all(x["p"] >= 0) and np.all(x["phi"] >= 0) and np.all(x["lam0"] > 0)
    if kind in ("no_process_noise", "precision_sum"):
        assert np.all(x["p"] == 0)
    if kind == "no_observation":
        assert np.all(x["phi"] == 0) and np.all(x["b"] == 0)
    if kind == "precision_sum":
        assert np.all(x["a"] == 1)
