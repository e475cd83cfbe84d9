"""Pin: the oracle reduces to independent library routines.

* The whole unsharded layer (t = 1) forward and backward equal the
  Hugging Face GPT2Block (pre-LayerNorm block, tanh GeLU "gelu_new",
  eps 1e-5, causal attention scaled by 1/sqrt(d), no dropout) run in
  float64 under torch autograd.
* The pieces equal torch's layer_norm, gelu(approximate="tanh") and
  scaled_dot_product_attention(is_causal=True).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from transformer_layer_step_b200 import synth


def _gpt2_block(h, a, f):
    from transformers import GPT2Config
    from transformers.models.gpt2.modeling_gpt2 import GPT2Block
    cfg = GPT2Config(n_embd=h, n_head=a, n_inner=f, resid_pdrop=0.0, attn_pdrop=0.0,
                     embd_pdrop=0.0, activation_function="gelu_new", layer_norm_epsilon=1e-5)
    cfg._attn_implementation = "eager"
    return GPT2Block(cfg, layer_idx=0).double().eval()


@pytest.mark.parametrize("b,s,h,a,f", [(2, 7, 16, 2, 64), (1, 12, 24, 3, 96)])
def test_layer_matches_hf_gpt2_block(b, s, h, a, f):
    rng = np.random.default_rng(7)
    T = b * s
    u = {
        "ln1_g": 1 + 0.1 * rng.standard_normal(h), "ln1_b": 0.1 * rng.standard_normal(h),
        "w_qkv": 0.2 * rng.standard_normal((3 * h, h)), "b_qkv": 0.1 * rng.standard_normal(3 * h),
        "w_o": 0.2 * rng.standard_normal((h, h)), "b_o": 0.1 * rng.standard_normal(h),
        "ln2_g": 1 + 0.1 * rng.standard_normal(h), "ln2_b": 0.1 * rng.standard_normal(h),
        "w_1": 0.2 * rng.standard_normal((f, h)), "b_1": 0.1 * rng.standard_normal(f),
        "w_2": 0.2 * rng.standard_normal((h, f)), "b_2": 0.1 * rng.standard_normal(h),
    }
    x = rng.standard_normal((T, h))
    r = rng.standard_normal((T, h))

    blk = _gpt2_block(h, a, f)
    with torch.no_grad():
        blk.ln_1.weight.copy_(torch.from_numpy(u["ln1_g"]))
        blk.ln_1.bias.copy_(torch.from_numpy(u["ln1_b"]))
        blk.attn.c_attn.weight.copy_(torch.from_numpy(u["w_qkv"].T))   # Conv1D is [in, out]
        blk.attn.c_attn.bias.copy_(torch.from_numpy(u["b_qkv"]))
        blk.attn.c_proj.weight.copy_(torch.from_numpy(u["w_o"].T))
        blk.attn.c_proj.bias.copy_(torch.from_numpy(u["b_o"]))
        blk.ln_2.weight.copy_(torch.from_numpy(u["ln2_g"]))
        blk.ln_2.bias.copy_(torch.from_numpy(u["ln2_b"]))
        blk.mlp.c_fc.weight.copy_(torch.from_numpy(u["w_1"].T))
        blk.mlp.c_fc.bias.copy_(torch.from_numpy(u["b_1"]))
        blk.mlp.c_proj.weight.copy_(torch.from_numpy(u["w_2"].T))
        blk.mlp.c_proj.bias.copy_(torch.from_numpy(u["b_2"]))
    xt = torch.from_numpy(x.reshape(b, s, h).copy()).requires_grad_(True)
    mask = torch.full((s, s), float("-inf"), dtype=torch.float64).triu(1)[None, None]
    yt = blk(xt, attention_mask=mask)
    yt = yt[0] if isinstance(yt, tuple) else yt
    (yt * torch.from_numpy(r.reshape(b, s, h))).sum().backward()

    dims = dict(b=b, s=s, h=h, a=a, f=f, t=1)
    p = synth.shard_params(u, 1)
    out, cache = oracle.layer_fwd(x, p, dims)
    dx, g = oracle.layer_bwd(cache, p, dims, r)
    gu = synth.unshard_params(g)

    np.testing.assert_allclose(out, yt.detach().numpy().reshape(T, h), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dx, xt.grad.numpy().reshape(T, h), rtol=0, atol=1e-11)
    lib = {
        "ln1_g": blk.ln_1.weight.grad, "ln1_b": blk.ln_1.bias.grad,
        "w_qkv": blk.attn.c_attn.weight.grad.T, "b_qkv": blk.attn.c_attn.bias.grad,
        "w_o": blk.attn.c_proj.weight.grad.T, "b_o": blk.attn.c_proj.bias.grad,
        "ln2_g": blk.ln_2.weight.grad, "ln2_b": blk.ln_2.bias.grad,
        "w_1": blk.mlp.c_fc.weight.grad.T, "b_1": blk.mlp.c_fc.bias.grad,
        "w_2": blk.mlp.c_proj.weight.grad.T, "b_2": blk.mlp.c_proj.bias.grad,
    }
    for name, ref in lib.items():
        np.testing.assert_allclose(gu[name], ref.numpy(), rtol=0, atol=1e-10, err_msg=name)


def test_pieces_match_torch_functional():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((9, 40)) * 3 + 1
    g = rng.standard_normal(40)
    b = rng.standard_normal(40)
    y, mu, rstd, xhat = oracle.layer_norm_fwd(x, g, b, 1e-5)
    ref = F.layer_norm(torch.from_numpy(x), (40,), torch.from_numpy(g), torch.from_numpy(b), 1e-5)
    np.testing.assert_allclose(y, ref.numpy(), rtol=0, atol=1e-12)

    z = np.linspace(-8, 8, 1001)
    np.testing.assert_allclose(oracle.gelu(z), F.gelu(torch.from_numpy(z), approximate="tanh").numpy(),
                               rtol=0, atol=1e-14)
    zt = torch.from_numpy(z).requires_grad_(True)
    F.gelu(zt, approximate="tanh").sum().backward()
    np.testing.assert_allclose(oracle.gelu_prime(z), zt.grad.numpy(), rtol=0, atol=1e-13)

    s, d = 11, 8
    q, k, v = (rng.standard_normal((s, d)) for _ in range(3))
    p, o = oracle.attention_head_fwd(q, k, v)
    ref = F.scaled_dot_product_attention(*(torch.from_numpy(a)[None, None] for a in (q, k, v)),
                                         is_causal=True)
    np.testing.assert_allclose(o, ref[0, 0].numpy(), rtol=0, atol=1e-13)


def test_layer_norm_backward_matches_autograd():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((6, 24))
    g = 1 + rng.standard_normal(24) * 0.3
    b = rng.standard_normal(24)
    gy = rng.standard_normal((6, 24))
    _, _, rstd, xhat = oracle.layer_norm_fwd(x, g, b, 1e-5)
    dx, dg, db = oracle.layer_norm_bwd(gy, xhat, rstd, g)
    xt = torch.from_numpy(x).requires_grad_(True)
    gt = torch.from_numpy(g).requires_grad_(True)
    bt = torch.from_numpy(b).requires_grad_(True)
    (F.layer_norm(xt, (24,), gt, bt, 1e-5) * torch.from_numpy(gy)).sum().backward()
    np.testing.assert_allclose(dx, xt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dg, gt.grad.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(db, bt.grad.numpy(), rtol=0, atol=1e-12)
    assert math.isfinite(float(dx.sum()))
