"""Pins for the oracle's layer stack (stack_fwd / stack_bwd).

* One layer: the stack is the layer, exactly.
* A layer with all linear weights zero passes its input through plus b_o and
  b_2, and passes dOut through exactly; placed on top of or below another
  layer, it fixes the order of the chain in both directions.
* Under a 16-bit precision the activation handed between layers (forward)
  and the gradient handed back (backward) are rounded once to the 16-bit
  type, the store between two layers.
* Finite differences of loss = sum(out * R) through two layers, for entries
  of the input and of each layer's weights.
"""
import numpy as np
import pytest

import oracle
from transformer_layer_step_b200 import synth

DIMS = dict(b=1, s=6, h=16, a=2, f=64, t=2)


def _params(rng, std=0.3, zero=False):
    h, f, t = DIMS["h"], DIMS["f"], DIMS["t"]
    u = {
        "ln1_g": 1 + 0.1 * rng.standard_normal(h), "ln1_b": 0.1 * rng.standard_normal(h),
        "w_qkv": std * rng.standard_normal((3 * h, h)), "b_qkv": 0.1 * rng.standard_normal(3 * h),
        "w_o": std * rng.standard_normal((h, h)), "b_o": 0.1 * rng.standard_normal(h),
        "ln2_g": 1 + 0.1 * rng.standard_normal(h), "ln2_b": 0.1 * rng.standard_normal(h),
        "w_1": std * rng.standard_normal((f, h)), "b_1": 0.1 * rng.standard_normal(f),
        "w_2": std * rng.standard_normal((h, f)), "b_2": 0.1 * rng.standard_normal(h),
    }
    if zero:
        for k in ("w_qkv", "w_o", "w_1", "w_2"):
            u[k] = np.zeros_like(u[k])
    return u, synth.shard_params(u, t)


def test_single_layer_stack_is_the_layer():
    rng = np.random.default_rng(1)
    _, p = _params(rng)
    x = rng.standard_normal((6, 16))
    g = rng.standard_normal((6, 16))
    out1, c1 = oracle.layer_fwd(x, p, DIMS)
    dx1, gr1 = oracle.layer_bwd(c1, p, DIMS, g)
    out, cs = oracle.stack_fwd(x, [p], DIMS)
    dx, gr = oracle.stack_bwd(cs, [p], DIMS, g)
    assert np.array_equal(out, out1) and np.array_equal(dx, dx1)
    assert all(np.array_equal(gr[0][k], gr1[k]) for k in gr1)


def test_zero_layer_fixes_the_chain_order():
    rng = np.random.default_rng(2)
    u0, p0 = _params(rng)
    uz, pz = _params(rng, zero=True)
    x = rng.standard_normal((6, 16))
    g = rng.standard_normal((6, 16))
    out0, c0 = oracle.layer_fwd(x, p0, DIMS)
    dx0, gr0 = oracle.layer_bwd(c0, p0, DIMS, g)
    # zero layer on top: its output is layer 0's plus its biases; dOut passes through
    out, cs = oracle.stack_fwd(x, [p0, pz], DIMS)
    np.testing.assert_allclose(out, out0 + uz["b_o"] + uz["b_2"], rtol=0, atol=1e-13)
    dx, gr = oracle.stack_bwd(cs, [p0, pz], DIMS, g)
    np.testing.assert_allclose(dx, dx0, rtol=1e-13, atol=1e-13)
    for k in gr0:
        np.testing.assert_allclose(gr[0][k], gr0[k], rtol=1e-12, atol=1e-13)
    # zero layer below: layer 0 sees the shifted input
    out, cs = oracle.stack_fwd(x, [pz, p0], DIMS)
    out_s, c_s = oracle.layer_fwd(x + uz["b_o"] + uz["b_2"], p0, DIMS)
    np.testing.assert_allclose(out, out_s, rtol=1e-13, atol=1e-13)
    dx, _ = oracle.stack_bwd(cs, [pz, p0], DIMS, g)
    dx_s, _ = oracle.layer_bwd(c_s, p0, DIMS, g)
    np.testing.assert_allclose(dx, dx_s, rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("prec", ["fp16", "bf16"])
def test_store_between_layers_under_a_precision(prec):
    rng = np.random.default_rng(3)
    u0, p0 = _params(rng)
    uz, pz = _params(rng, zero=True)
    x = oracle.optim.round_to_16(rng.standard_normal((6, 16)), prec)
    g = rng.standard_normal((6, 16))                 # not on the 16-bit grid
    out0, c0 = oracle.layer_fwd(x, p0, DIMS, precision=prec)
    out, cs = oracle.stack_fwd(x, [p0, pz], DIMS, precision=prec)
    # the zero layer's residual path is fp32-exact, so only the store between
    # the layers rounds layer 0's output
    np.testing.assert_allclose(out, oracle.optim.round_to_16(out0, prec) + uz["b_o"] + uz["b_2"],
                               rtol=0, atol=1e-13)
    assert not np.allclose(out, out0 + uz["b_o"] + uz["b_2"], rtol=0, atol=1e-13)
    dx, _ = oracle.stack_bwd(cs, [p0, pz], DIMS, g)
    dx0, _ = oracle.layer_bwd(c0, p0, DIMS, oracle.optim.round_to_16(g, prec))
    np.testing.assert_allclose(dx, dx0, rtol=1e-12, atol=1e-13)


def test_two_layer_stack_matches_finite_differences():
    rng = np.random.default_rng(4)
    _, p0 = _params(rng)
    _, p1 = _params(rng)
    ps = [p0, p1]
    x = rng.standard_normal((6, 16))
    r = rng.standard_normal((6, 16))

    def loss():
        out, _ = oracle.stack_fwd(x, ps, DIMS)
        return float((out * r).sum())

    _, cs = oracle.stack_fwd(x, ps, DIMS)
    dx, grads = oracle.stack_bwd(cs, ps, DIMS, r)
    eps = 1e-6
    checks = [(x, dx, (2, 5)), (x, dx, (5, 0)),
              (p0["w_qkv"], grads[0]["w_qkv"], (1, 7, 3)), (p0["w_2"], grads[0]["w_2"], (0, 4, 9)),
              (p1["w_1"], grads[1]["w_1"], (1, 3, 11)), (p1["ln1_g"], grads[1]["ln1_g"], (6,)),
              (p0["b_o"], grads[0]["b_o"], (13,))]
    for arr, g, idx in checks:
        old = arr[idx]
        arr[idx] = old + eps
        lp = loss()
        arr[idx] = old - eps
        lm = loss()
        arr[idx] = old
        fd = (lp - lm) / (2 * eps)
        assert abs(fd - g[idx]) <= 1e-6 * max(1.0, abs(fd)), (idx, fd, g[idx])
