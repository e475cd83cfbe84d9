"""GPU parity of the fused causal attention forward (gptl_attention_fwd)
against the oracle's attention head, computed exactly from the same 16-bit
Q, K, V: O within a 16-bit storage tolerance, and each row's base-2
log-sum-exp of the scaled scores (which the backward uses to recompute P).

Shapes cover head_dim 32, 64, 80 and 128, sequences below one 128-row
block, several blocks and a ragged last block, and tp 1, 2, 4."""
import math

import numpy as np
import pytest
import torch

import oracle
from transformer_layer_step_b200 import gptlayer as G
from gpu_util import need_gpu, dev_tensor, host_values, rounded, stream, check_device_error

pytestmark = pytest.mark.gpu

CASES = [
    # batch, seq, hidden, heads, tp, dtype
    (2, 64, 128, 4, 2, "fp16"),      # head_dim 32, one partial block
    (1, 384, 640, 8, 4, "fp16"),     # head_dim 80, three blocks
    (2, 256, 256, 4, 1, "bf16"),     # head_dim 64
    (1, 272, 512, 4, 1, "bf16"),     # head_dim 128, ragged last block
]


@pytest.mark.parametrize("b,s,h,a,t,dtype", CASES)
def test_attention_fwd(b, s, h, a, t, dtype):
    need_gpu()
    d, hs, as_ = h // a, h // t, a // t
    rng = np.random.default_rng(s + h)
    qkv = rounded(rng.standard_normal((t, b * s, 3 * hs)), dtype)
    qkv_t = dev_tensor(qkv, dtype)
    tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
    o = torch.full((t, b * s, hs), float("nan"), dtype=tdt, device="cuda")
    lse = torch.full((t * b * as_, s), float("nan"), dtype=torch.float32, device="cuda")
    G.attention_fwd(b, s, h, a, t, dtype, qkv_t, o, lse, stream())
    check_device_error()
    o_got = host_values(o, dtype)
    lse_got = lse.cpu().numpy()
    # each probability enters P V as a 16-bit value (relative error <= u), so
    # O moves by at most u * max|V| before its own rounding (<= u |O|)
    u = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -11
    for i in range(t):
        for j in range(b):
            rows = slice(j * s, (j + 1) * s)
            for eta in range(as_):
                cols = slice(eta * d, (eta + 1) * d)
                q = qkv[i, rows, 0 * hs:1 * hs][:, cols]
                k = qkv[i, rows, 1 * hs:2 * hs][:, cols]
                v = qkv[i, rows, 2 * hs:3 * hs][:, cols]
                _, o_ref = oracle.attention_head_fwd(q, k, v)
                np.testing.assert_allclose(o_got[i, rows, cols], o_ref, rtol=2 * u,
                                           atol=2 * u * float(np.abs(v).max()))
                z = (q @ k.T) / math.sqrt(d)
                z = np.where(np.tril(np.ones((s, s), bool)), z, -np.inf)
                zmax = z.max(axis=1)
                lse_ref = (zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))) / math.log(2.0)
                g = (i * b + j) * as_ + eta
                np.testing.assert_allclose(lse_got[g], lse_ref, rtol=1e-5, atol=1e-4)


def test_attention_fwd_is_deterministic():
    need_gpu()
    b, s, h, a, t, dtype = 2, 256, 256, 4, 1, "bf16"
    hs, as_ = h // t, a // t
    rng = np.random.default_rng(1)
    qkv_t = dev_tensor(rounded(rng.standard_normal((t, b * s, 3 * hs)), dtype), dtype)
    outs = []
    for _ in range(2):
        o = torch.zeros((t, b * s, hs), dtype=torch.bfloat16, device="cuda")
        lse = torch.zeros((t * b * as_, s), dtype=torch.float32, device="cuda")
        G.attention_fwd(b, s, h, a, t, dtype, qkv_t, o, lse, stream())
        outs.append((o, lse))
    check_device_error()
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def _attention_bwd_exact(q, k, v, do, dtype):
    """Per-head backward in float64 with P taken in the 16-bit type, the
    method's reading (P enters the products as a 16-bit operand)."""
    s, d = q.shape
    z = (q @ k.T) / math.sqrt(d)
    z = np.where(np.tril(np.ones((s, s), bool)), z, -np.inf)
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    o = p @ v
    p16 = rounded(p, dtype)
    dp = do @ v.T
    drow = (do * o).sum(axis=1, keepdims=True)
    ds = p16 * (dp - drow) / math.sqrt(d)
    return ds @ k, ds.T @ q, p16.T @ do


@pytest.mark.parametrize("b,s,h,a,t,dtype", CASES)
def test_attention_bwd(b, s, h, a, t, dtype):
    need_gpu()
    d, hs, as_ = h // a, h // t, a // t
    rng = np.random.default_rng(7 * s + h)
    qkv = rounded(rng.standard_normal((t, b * s, 3 * hs)), dtype)
    dout = rounded(rng.standard_normal((t, b * s, hs)), dtype)
    tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
    qkv_t, dout_t = dev_tensor(qkv, dtype), dev_tensor(dout, dtype)
    o = torch.zeros((t, b * s, hs), dtype=tdt, device="cuda")
    lse = torch.zeros((t * b * as_, s), dtype=torch.float32, device="cuda")
    G.attention_fwd(b, s, h, a, t, dtype, qkv_t, o, lse, stream())
    dvec = torch.zeros_like(lse)
    dqkv = torch.full((t, b * s, 3 * hs), float("nan"), dtype=tdt, device="cuda")
    G.attention_bwd(b, s, h, a, t, dtype, qkv_t, o, dout_t, lse, dvec, dqkv, stream())
    check_device_error()
    got = host_values(dqkv, dtype)
    o_used = host_values(o, dtype)
    u = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -11
    for i in range(t):
        for j in range(b):
            rows = slice(j * s, (j + 1) * s)
            for eta in range(as_):
                cols = slice(eta * d, (eta + 1) * d)
                q = qkv[i, rows, 0 * hs:1 * hs][:, cols]
                k = qkv[i, rows, 1 * hs:2 * hs][:, cols]
                v = qkv[i, rows, 2 * hs:3 * hs][:, cols]
                do = dout[i, rows, cols]
                dq, dk, dv = _attention_bwd_exact(q, k, v, do, dtype)
                # the kernel forms D from the stored 16-bit O; the reference
                # from the exact O: both are dO . O up to one rounding of O
                for name, got_part, ref in (("dq", got[i, rows, 0 * hs:1 * hs][:, cols], dq),
                                            ("dk", got[i, rows, 1 * hs:2 * hs][:, cols], dk),
                                            ("dv", got[i, rows, 2 * hs:3 * hs][:, cols], dv)):
                    scale = float(np.abs(ref).max())
                    err = float(np.abs(got_part - ref).max())
                    assert err <= 16 * u * scale, (name, i, j, eta, err, scale)
    assert np.all(np.isfinite(o_used))
