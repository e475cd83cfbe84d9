"""GPU parity of the fused causal attention (gptl_attention_fwd,
gptl_attention_bwd) against the oracle's attention head on the same 16-bit
Q, K, V (and dO, O for the backward).

Forward: O against the method's own result, round(P16 V) with P16 the
normalised probabilities rounded to the 16-bit type (the fused softmax's
output, "Training GPT-2 with Megatron-LM" §6.2): apart by at most one
16-bit step of O and of each P16 anywhere, and equal bit for bit in at
least 99 % of the elements (a
kernel that rounded anything but the normalised P, such as a single pass that
rounds exp(S - running max) and divides at the end, moves far more of them);
and each row's base-2 log-sum-exp of the scaled scores (which the backward
uses to recompute P).

Backward: dQ, dK, dV against oracle.attention_head_bwd at the method's
precision, given the same P16, dO and the O the kernel reads.

Shapes cover head_dim 32, 64, 80 and 128, sequences below one 128-row
block, several blocks and a ragged last block, tp 1, 2, 4, and a shard of
64 heads / 8192 columns (the row-term kernel walks it in chunks)."""
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
    (1, 128, 8192, 64, 1, "bf16"),   # 64 heads, 8192 columns per shard
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
    # u: the 16-bit type's relative half step; one step is at most 2u |O|
    u = 2.0 ** -8 if dtype == "bf16" else 2.0 ** -11
    same = total = 0
    for i in range(t):
        for j in range(b):
            rows = slice(j * s, (j + 1) * s)
            for eta in range(as_):
                cols = slice(eta * d, (eta + 1) * d)
                q = qkv[i, rows, 0 * hs:1 * hs][:, cols]
                k = qkv[i, rows, 1 * hs:2 * hs][:, cols]
                v = qkv[i, rows, 2 * hs:3 * hs][:, cols]
                p16, o_ref = oracle.attention_head_fwd(q, k, v, precision=dtype)
                o_ref = rounded(o_ref, dtype)
                got_h = o_got[i, rows, cols]
                # one 16-bit step of O, plus one step of any P16 whose exact value
                # sat within the kernel's ex2 error of a rounding midpoint (rows
                # with few keys have P near 1), plus the fp32 accumulation of P V
                bound = (2 * u * np.maximum(np.abs(o_ref), np.abs(got_h)) + 2 * u * (p16 @ np.abs(v))
                         + 2.0 ** -14 * float(np.abs(v).max()))
                assert np.all(np.abs(got_h - o_ref) <= bound), float(np.abs(got_h - o_ref).max())
                same += int(np.sum(got_h == o_ref))
                total += got_h.size
                z = (q @ k.T) / math.sqrt(d)
                z = np.where(np.tril(np.ones((s, s), bool)), z, -np.inf)
                zmax = z.max(axis=1)
                lse_ref = (zmax + np.log(np.exp(z - zmax[:, None]).sum(axis=1))) / math.log(2.0)
                g = (i * b + j) * as_ + eta
                np.testing.assert_allclose(lse_got[g], lse_ref, rtol=1e-5, atol=1e-4)
    assert same >= 0.99 * total, (same, total)


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
    dpart = torch.full((b * ((s + 31) // 32) * 3 * h,), float("nan"), device="cuda")
    dbias = torch.full((t, 3 * hs), float("nan"), device="cuda")
    G.attention_bwd(b, s, h, a, t, dtype, qkv_t, o, dout_t, lse, dvec, dqkv, dpart, dbias,
                    stream=stream())
    check_device_error()
    got = host_values(dqkv, dtype)
    # the bias gradient that the kernels sum as they store dQ, dK, dV: the
    # column sums of the stored values, per shard (fp32 sums of 32 rows, then
    # of the partial rows)
    want = got.astype(np.float64).sum(axis=1)
    db = dbias.cpu().numpy().astype(np.float64)
    bound = 4e-6 * np.abs(got).astype(np.float64).sum(axis=1) + 1e-30
    assert np.all(np.abs(db - want) <= bound), float(np.max(np.abs(db - want) / bound))
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
                p16, _ = oracle.attention_head_fwd(q, k, v, precision=dtype)
                dq, dk, dv = oracle.attention_head_bwd(q, k, v, p16, do, o_used[i, rows, cols],
                                                       precision=dtype)
                for name, got_part, ref in (("dq", got[i, rows, 0 * hs:1 * hs][:, cols], dq),
                                            ("dk", got[i, rows, 1 * hs:2 * hs][:, cols], dk),
                                            ("dv", got[i, rows, 2 * hs:3 * hs][:, cols], dv)):
                    scale = float(np.abs(ref).max())
                    err = float(np.abs(got_part - ref).max())
                    assert err <= 16 * u * scale, (name, i, j, eta, err, scale)
    assert np.all(np.isfinite(o_used))
