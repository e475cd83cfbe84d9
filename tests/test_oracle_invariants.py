"""Pins: invariants and closed forms of the oracle's layer.

* The tensor-parallel forward (t = 2, 4) equals the unsharded forward
  (t = 1) built from the same unsharded weights, and the re-assembled
  gradients agree (the TP split is exact algebra: "Megatron-LM 3D
  parallelism", §1).
* Causal softmax rows sum to 1, carry exactly zero mass above the diagonal,
  and row 0 is [1, 0, ...].
* With W_q = 0 and b_q = 0 every score is equal, so each output row is the
  running mean of the value rows; with seq 1, O = V.
* LayerNorm of a constant row is beta; with gamma 1, beta 0 every row has
  mean 0 and variance var/(var + eps).
* GeLU: gelu(0) = 0, gelu(z) - gelu(-z) = z, gelu(z) - z -> 0 as z grows,
  within 1e-3 of the exact z*Phi(z), derivative equal to its finite
  difference.
* All linear weights 0: Out = X + b_o + b_2 and dX = dOut exactly.
"""
import math

import numpy as np
import pytest
from scipy.special import erf

import oracle
from transformer_layer_step_b200 import synth


def _unsharded(rng, h, f, std=0.05, bias=0.05):
    return {
        "ln1_g": 1 + bias * rng.standard_normal(h), "ln1_b": bias * rng.standard_normal(h),
        "w_qkv": std * rng.standard_normal((3 * h, h)), "b_qkv": bias * rng.standard_normal(3 * h),
        "w_o": std * rng.standard_normal((h, h)), "b_o": bias * rng.standard_normal(h),
        "ln2_g": 1 + bias * rng.standard_normal(h), "ln2_b": bias * rng.standard_normal(h),
        "w_1": std * rng.standard_normal((f, h)), "b_1": bias * rng.standard_normal(f),
        "w_2": std * rng.standard_normal((h, f)), "b_2": bias * rng.standard_normal(h),
    }


@pytest.mark.parametrize("t", [2, 4])
def test_sharded_equals_unsharded(t):
    rng = np.random.default_rng(11)
    b, s, h, a, f = 2, 9, 32, 4, 128
    u = _unsharded(rng, h, f)
    x = rng.standard_normal((b * s, h))
    r = rng.standard_normal((b * s, h))
    d1 = dict(b=b, s=s, h=h, a=a, f=f, t=1)
    dt = dict(d1, t=t)
    p1, pt = synth.shard_params(u, 1), synth.shard_params(u, t)
    o1, c1 = oracle.layer_fwd(x, p1, d1)
    ot, ct = oracle.layer_fwd(x, pt, dt)
    assert np.abs(o1 - ot).max() <= 1e-12 * np.abs(o1).max()
    dx1, g1 = oracle.layer_bwd(c1, p1, d1, r)
    dxt, gt = oracle.layer_bwd(ct, pt, dt, r)
    assert np.abs(dx1 - dxt).max() <= 1e-12 * np.abs(dx1).max()
    gu1, gut = synth.unshard_params(g1), synth.unshard_params(gt)
    for k in gu1:
        assert np.abs(gu1[k] - gut[k]).max() <= 1e-12 * max(np.abs(gu1[k]).max(), 1e-300), k


def test_shard_layout_round_trip():
    rng = np.random.default_rng(0)
    u = _unsharded(rng, 16, 64)
    for t in (1, 2, 4):
        back = synth.unshard_params(synth.shard_params(u, t))
        for k in u:
            np.testing.assert_array_equal(back[k], u[k])
    # shard i of W_qkv holds the Q, K, V rows of its own heads
    w = np.arange(3 * 8)[:, None] * np.ones((1, 2))
    ws = synth.shard_qkv_rows(w, 2)
    assert list(ws[1][:, 0]) == [4, 5, 6, 7, 12, 13, 14, 15, 20, 21, 22, 23]


def test_causal_softmax_invariants():
    rng = np.random.default_rng(2)
    z = rng.standard_normal((17, 17)) * 4
    p = oracle.causal_softmax(z)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(p[np.triu_indices(17, 1)] == 0.0)
    assert p[0, 0] == 1.0 and np.all(p[0, 1:] == 0.0)
    assert np.all(p[np.tril_indices(17)] > 0)
    # worked example: scores 0, ln 2, ln 3 on row 2 -> 1/6, 2/6, 3/6
    z3 = np.zeros((3, 3))
    z3[2] = [0.0, math.log(2.0), math.log(3.0)]
    np.testing.assert_allclose(oracle.causal_softmax(z3)[2], [1 / 6, 2 / 6, 3 / 6], atol=1e-15)


def test_layer_probabilities_are_causal():
    cfg = synth.CONFIGS["tiny"]
    inp = synth.make_inputs(cfg, variant="biased")
    x = synth.from_bits(inp["x"], cfg.dtype)
    p = {k: synth.from_bits(v, cfg.dtype) for k, v in inp["params"].items()}
    _, cache = oracle.layer_fwd(x, p, cfg.dims())
    pr = cache["probs"]
    np.testing.assert_allclose(pr.sum(axis=-1), 1.0, atol=1e-12)
    iu = np.triu_indices(cfg.seq, 1)
    assert np.all(pr[..., iu[0], iu[1]] == 0.0)


def test_uniform_attention_is_running_mean():
    rng = np.random.default_rng(4)
    b, s, h, a, f, t = 2, 6, 16, 2, 64, 2
    u = _unsharded(rng, h, f)
    u["w_qkv"][:h] = 0.0          # W_q = 0
    u["b_qkv"][:h] = 0.0
    x = rng.standard_normal((b * s, h))
    dims = dict(b=b, s=s, h=h, a=a, f=f, t=t)
    _, cache = oracle.layer_fwd(x, synth.shard_params(u, t), dims)
    hs = h // t
    for i in range(t):
        v = cache["c"][i][:, 2 * hs:]
        for j in range(b):
            vj = v[j * s:(j + 1) * s]
            running = np.cumsum(vj, axis=0) / np.arange(1, s + 1)[:, None]
            np.testing.assert_allclose(cache["o"][i][j * s:(j + 1) * s], running, atol=1e-13)


def test_single_position_attention_is_identity():
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((1, 8)) for _ in range(3))
    p, o = oracle.attention_head_fwd(q, k, v)
    assert p[0, 0] == 1.0
    np.testing.assert_array_equal(o, v)


def test_layer_norm_closed_forms():
    g = np.linspace(0.5, 2, 10)
    b = np.linspace(-1, 1, 10)
    y, _, _, _ = oracle.layer_norm_fwd(np.full((3, 10), 4.25), g, b, 1e-5)
    np.testing.assert_allclose(y, np.broadcast_to(b, (3, 10)), atol=1e-15)
    rng = np.random.default_rng(6)
    x = rng.standard_normal((5, 64)) * 0.01     # small variance: eps matters
    y, _, _, _ = oracle.layer_norm_fwd(x, np.ones(64), np.zeros(64), 1e-5)
    var = x.var(axis=1)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-14)
    np.testing.assert_allclose(y.var(axis=1), var / (var + 1e-5), rtol=1e-12)


def test_gelu_closed_forms():
    z = np.linspace(-6, 6, 241)
    assert oracle.gelu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(oracle.gelu(z) - oracle.gelu(-z), z, atol=1e-14)
    big = np.array([10.0, 20.0, 40.0])
    np.testing.assert_allclose(oracle.gelu(big), big, rtol=1e-15)
    exact = 0.5 * z * (1 + erf(z / math.sqrt(2)))
    assert np.abs(oracle.gelu(z) - exact).max() < 1e-3
    e = 1e-6
    np.testing.assert_allclose(oracle.gelu_prime(z), (oracle.gelu(z + e) - oracle.gelu(z - e)) / (2 * e),
                               atol=1e-8)


def test_zero_weights_layer():
    rng = np.random.default_rng(8)
    b, s, h, a, f, t = 2, 5, 16, 4, 64, 2
    u = _unsharded(rng, h, f)
    for k in ("w_qkv", "w_o", "w_1", "w_2"):
        u[k] = np.zeros_like(u[k])
    x = rng.standard_normal((b * s, h))
    dims = dict(b=b, s=s, h=h, a=a, f=f, t=t)
    p = synth.shard_params(u, t)
    out, cache = oracle.layer_fwd(x, p, dims)
    np.testing.assert_allclose(out, x + u["b_o"] + u["b_2"], atol=1e-14)
    g = rng.standard_normal((b * s, h))
    dx, _ = oracle.layer_bwd(cache, p, dims, g)
    np.testing.assert_array_equal(dx, g)
