"""Pins for the optimizer side of the oracle.

* Loss-scale rule: hand-computed transition sequences stored in
  tests/golden/loss_scale_sequences.txt (derivation in its header).
* Overflow check: brute-force scan of the same buffer with inf and NaN
  planted at the first, last, random and shard-boundary positions.
* Adam: at t = 1 the bias-corrected moments are g and g^2, so
  dp = -lr * g / (|g| + eps); with a constant gradient every step moves by
  that same amount; multi-step random gradients equal torch.optim.AdamW in
  float64 (decoupled weight decay); a skipped step leaves everything
  bit-identical.
* 16-bit cast: bf16 round-to-nearest-even equals torch's fp32 -> bf16
  conversion on fp32 inputs; halfway cases round to even.
"""
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "loss_scale_sequences.txt")
HP = dict(growth_interval=1000, growth_factor=2.0, backoff_factor=0.5, min_scale=1.0)


def _golden_rows():
    rows = []
    with open(GOLDEN) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            a, flags, b = (part.strip() for part in line.split("|"))
            s0, k0, st0 = a.split()
            seq = []
            for item in flags.split(","):
                n, val = item.split("x")
                seq += [int(val)] * int(n)
            s1, k1, st1 = b.split()
            rows.append(((float(s0), int(k0), int(st0)), seq, (float(s1), int(k1), int(st1))))
    return rows


@pytest.mark.parametrize("row", _golden_rows())
def test_loss_scale_golden(row):
    (s0, k0, st0), seq, (s1, k1, st1) = row
    st = dict(scale=s0, growth_tracker=k0, step=st0)
    for f in seq:
        st = oracle.loss_scale_update(st, f, **HP)
    assert (st["scale"], st["growth_tracker"], st["step"]) == (s1, k1, st1)


def test_found_inf_brute_force():
    rng = np.random.default_rng(0)
    g = rng.standard_normal(10_000).astype(np.float32)
    assert oracle.found_inf(g) == 0
    for pos in (0, 9_999, 1234, 2_500, 5_000, 7_500):
        for bad in (np.inf, -np.inf, np.nan):
            h = g.copy()
            h[pos] = bad
            brute = int(any(not np.isfinite(v) for v in h))
            assert oracle.found_inf(h) == brute == 1
    big = np.float32(3.0e38)
    assert oracle.found_inf(np.array([big, -big], dtype=np.float32)) == 0
    assert oracle.found_inf(g[:10], np.array([np.nan], dtype=np.float32)) == 1


def test_adam_first_step_closed_form():
    rng = np.random.default_rng(1)
    n = 4096
    p0 = rng.standard_normal(n).astype(np.float32) * 0.02
    g = rng.standard_normal(n).astype(np.float32) * 1e-3
    scale = 1024.0
    lr, eps = 6e-5, 1e-8
    p1, m1, v1, w16 = oracle.adam_step(p0, np.zeros(n), np.zeros(n), g * scale, scale, 0,
                                       lr, 0.9, 0.95, eps, 0.0, "bf16", 0)
    gg = g.astype(np.float64)
    np.testing.assert_allclose(p1, p0 - lr * gg / (np.abs(gg) + eps), rtol=1e-13, atol=1e-20)
    np.testing.assert_allclose(m1, 0.1 * gg, rtol=1e-14)
    np.testing.assert_allclose(v1, 0.05 * gg * gg, rtol=1e-14)


def test_adam_constant_gradient_closed_form():
    g = np.array([1e-3, -2e-2, 5e-7, -3.0])
    p = np.array([0.1, -0.2, 0.0, 1.0])
    m = np.zeros(4)
    v = np.zeros(4)
    lr, eps = 1e-3, 1e-8
    for step in range(25):
        p, m, v, _ = oracle.adam_step(p, m, v, g, 1.0, step, lr, 0.9, 0.95, eps, 0.0, "fp16", 0)
    expect = np.array([0.1, -0.2, 0.0, 1.0]) - 25 * lr * g / (np.abs(g) + eps)
    np.testing.assert_allclose(p, expect, rtol=1e-10, atol=1e-15)


def test_adam_matches_torch_adamw():
    rng = np.random.default_rng(2)
    n = 513
    p0 = rng.standard_normal(n) * 0.02
    hp = dict(lr=6e-5, betas=(0.9, 0.95), eps=1e-8, weight_decay=0.1)
    pt = torch.tensor(p0, dtype=torch.float64, requires_grad=True)
    opt = torch.optim.AdamW([pt], **hp)
    p, m, v = p0.copy(), np.zeros(n), np.zeros(n)
    scale = 4096.0
    for step in range(6):
        g = rng.standard_normal(n) * 1e-2
        pt.grad = torch.tensor(g, dtype=torch.float64)
        opt.step()
        p, m, v, _ = oracle.adam_step(p, m, v, g * scale, scale, step, hp["lr"], 0.9, 0.95,
                                      hp["eps"], hp["weight_decay"], "bf16", 0)
    np.testing.assert_allclose(p, pt.detach().numpy(), rtol=1e-12, atol=1e-18)


def test_adam_skip_is_identity():
    p = np.arange(5, dtype=np.float32)
    m = np.ones(5, dtype=np.float32)
    v = np.ones(5, dtype=np.float32)
    g = np.array([1, np.inf, 0, 0, 0], dtype=np.float32)
    p1, m1, v1, w = oracle.adam_step(p, m, v, g, 1.0, 3, 1e-3, 0.9, 0.95, 1e-8, 0.0, "fp16", 1)
    assert w is None and p1 is p and m1 is m and v1 is v


def test_cast_to_16():
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(20_000) * 10.0 ** rng.integers(-30, 30, 20_000)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.cast_to_16(x.astype(np.float64), "bf16"), ref)
    # halfway cases round to the even neighbour
    half = np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)])
    np.testing.assert_array_equal(oracle.cast_to_16(half, "bf16"),
                                  np.array([0x3F80, 0x3F82, 0xBF80], dtype=np.uint16))
    # just above halfway rounds up
    assert oracle.cast_to_16(np.array([1 + 2.0 ** -8 + 2.0 ** -30]), "bf16")[0] == 0x3F81
    np.testing.assert_array_equal(oracle.cast_to_16(np.array([1 + 2.0 ** -11]), "fp16"),
                                  np.array([0x3C00], dtype=np.uint16))
