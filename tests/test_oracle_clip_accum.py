"""Pins for the oracle's gradient clipping and gradient accumulation.

* grad_norm: closed forms (a 3-4-5 gradient, n equal entries) on the
  scaled fp32 arena, so that a missing unscale, a missing square root or an
  absolute-value sum fails.
* clip_coefficient: exactly 1 at or below the threshold's reach, and the
  clipped gradient's norm equal to max_norm up to the 1e-6 guard.
* Adam with clipping: several steps, some clipped and some not, equal
  torch.nn.utils.clip_grad_norm_ followed by torch.optim.AdamW in float64
  (the library's own global-norm clip, computed independently).
* accumulate: bit-equal to torch's fp32 addition, including operands whose
  exponents are far apart; and the semantic pin: the layer's weight
  gradients of a two-sequence batch equal the sum of the two one-sequence
  batches' gradients (the loss is a sum over tokens, so accumulating
  micro-batches is summing their gradients).
"""
import math

import numpy as np
import torch

import oracle
from transformer_layer_step_b200 import synth


def test_grad_norm_closed_forms():
    S = 65536.0
    g = np.zeros(1000, dtype=np.float32)
    g[17], g[901] = 3 * S, -4 * S
    assert oracle.grad_norm(g, S) == 5.0
    n, c = 1 << 20, 1e-3
    g = np.full(n, c * 1024.0, dtype=np.float32)
    assert abs(oracle.grad_norm(g, 1024.0) - float(np.float32(c * 1024.0)) / 1024.0 * math.sqrt(n)) \
        <= 1e-12 * c * math.sqrt(n)
    # a power-of-two rescale of both the arena and the scale is exact
    rng = np.random.default_rng(5)
    g = (rng.standard_normal(4097) * 1e-2).astype(np.float32)
    assert oracle.grad_norm(g, 1.0) == oracle.grad_norm(g * np.float32(8.0), 8.0)


def test_clip_coefficient():
    assert oracle.clip_coefficient(0.5, 1.0) == 1.0
    assert oracle.clip_coefficient(0.0, 1.0) == 1.0
    # at the threshold the 1e-6 guard clips by a hair, as the usual rule does
    c = oracle.clip_coefficient(1.0, 1.0)
    assert 1.0 - 2e-6 < c < 1.0
    rng = np.random.default_rng(6)
    g = (rng.standard_normal(5000) * 0.3).astype(np.float64)
    norm = float(np.sqrt((g * g).sum()))
    for max_norm in (0.25, 1.0, 3.0):
        cc = oracle.clip_coefficient(norm, max_norm)
        clipped = oracle.grad_norm(g * cc, 1.0)
        assert abs(clipped - max_norm) <= 1e-6 * max_norm + 1e-12
        # the direction is kept
        assert np.allclose(g * cc / clipped, g / norm, rtol=1e-12, atol=0)


def test_clipped_adam_matches_torch():
    rng = np.random.default_rng(7)
    n = 777
    p0 = rng.standard_normal(n) * 0.02
    hp = dict(lr=6e-5, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    max_norm = 1.0
    pt = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([pt], **hp)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    scale = 2048.0
    clipped_steps = 0
    for step, mag in enumerate([0.5, 0.01, 0.2, 0.001, 1.0, 0.03]):
        g = rng.standard_normal(n) * mag                  # norm ~ mag * sqrt(n)
        pt.grad = torch.tensor(g, dtype=torch.float64)
        torch.nn.utils.clip_grad_norm_([pt], max_norm)
        opt.step()
        norm = oracle.grad_norm(g * scale, scale)
        cc = oracle.clip_coefficient(norm, max_norm)
        clipped_steps += cc < 1.0
        p, m, v, _ = oracle.adam_step(p, m, v, g * scale, scale, step, hp["lr"], 0.9, 0.95,
                                      hp["eps"], hp["weight_decay"], "bf16", 0, clip_coef=cc)
    assert 2 <= clipped_steps < 6
    np.testing.assert_allclose(p, pt.detach().numpy(), rtol=1e-12, atol=1e-18)


def test_accumulate_is_fp32_addition():
    rng = np.random.default_rng(8)
    a = (rng.standard_normal(20000) * 10.0 ** rng.integers(-20, 20, 20000)).astype(np.float32)
    b = (rng.standard_normal(20000) * 10.0 ** rng.integers(-20, 20, 20000)).astype(np.float32)
    b[:10] = -a[:10]                                   # exact cancellation
    b[10:20] = a[10:20] * np.float32(2.0 ** -24)      # addends near half an ulp
    want = (torch.from_numpy(a) + torch.from_numpy(b)).numpy()
    got = oracle.accumulate(a, b)
    assert got.dtype == np.float32
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))


def test_accumulated_microbatch_gradients_equal_the_batch_gradient():
    rng = np.random.default_rng(9)
    s, h, a, f, t = 7, 32, 4, 128, 2
    u = {
        "ln1_g": 1 + 0.05 * rng.standard_normal(h), "ln1_b": 0.05 * rng.standard_normal(h),
        "w_qkv": 0.05 * rng.standard_normal((3 * h, h)), "b_qkv": 0.05 * rng.standard_normal(3 * h),
        "w_o": 0.05 * rng.standard_normal((h, h)), "b_o": 0.05 * rng.standard_normal(h),
        "ln2_g": 1 + 0.05 * rng.standard_normal(h), "ln2_b": 0.05 * rng.standard_normal(h),
        "w_1": 0.05 * rng.standard_normal((f, h)), "b_1": 0.05 * rng.standard_normal(f),
        "w_2": 0.05 * rng.standard_normal((h, f)), "b_2": 0.05 * rng.standard_normal(h),
    }
    params = synth.shard_params(u, t)
    x = rng.standard_normal((2 * s, h))
    r = rng.standard_normal((2 * s, h))
    d2 = dict(b=2, s=s, h=h, a=a, f=f, t=t)
    d1 = dict(d2, b=1)
    _, c2 = oracle.layer_fwd(x, params, d2)
    _, g2 = oracle.layer_bwd(c2, params, d2, r)
    acc = None
    for j in range(2):
        rows = slice(j * s, (j + 1) * s)
        _, c1 = oracle.layer_fwd(x[rows], params, d1)
        _, g1 = oracle.layer_bwd(c1, params, d1, r[rows])
        acc = g1 if acc is None else {k: acc[k] + g1[k] for k in acc}
    for k in g2:
        assert np.abs(acc[k] - g2[k]).max() <= 1e-12 * max(np.abs(g2[k]).max(), 1e-300), k
