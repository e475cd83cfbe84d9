"""GPU checks of the layer stack (gpt_stack_fwd / gpt_stack_bwd through the
C ABI, and one optimizer call over every layer's parameters).

* Composition, bit for bit: each layer of the stack gives exactly what the
  single-layer step gives on the same input (the stored output of the layer
  below, or the stored input gradient of the layer above), in both
  directions.  The kernels are deterministic, so any plumbing mistake (a
  wrong buffer, offset or order) shows as a mismatch.
* Parity with the oracle's stack (fp16) for the output, dX and every
  layer's gradients, each within the layer test's 2e-2 * RMS bar.
* The optimizer call covers the whole arena: every layer's block matches
  the oracle's Adam.
"""
import dataclasses

import numpy as np
import torch

import oracle
from transformer_layer_step_b200 import synth
from transformer_layer_step_b200.harness import LayerStack, LayerStep, tensor_to_bits
from gpu_util import need_gpu, host_values, check_device_error, rel_max_err
import pytest

pytestmark = pytest.mark.gpu

CFG = synth.CONFIGS["tiny"]          # fp16, batch 2, seq 64, hidden 128, 4 heads, ffn 512, tp 2
N_LAYERS = 3


def _inputs():
    layers = [synth.make_inputs(CFG, seed=10 + l, variant="biased") for l in range(N_LAYERS)]
    first = synth.make_inputs(CFG, seed=3, variant="biased", with_r=True)
    return [d["params"] for d in layers], first["x"], first["r"]


def test_stack_is_the_composition_of_single_layers():
    need_gpu()
    params, x_bits, r_bits = _inputs()
    st = LayerStack(CFG, params, x_bits)
    dy_bits = synth.loss_grad_bits(CFG, st.hyper["init_scale"], r_bits)
    st.set_dy_bits(dy_bits)
    st.fwd()
    st.bwd()
    check_device_error()
    acts = [tensor_to_bits(st.acts[l]) for l in range(N_LAYERS)]
    # forward: layer l on the stored output of layer l-1
    inp = x_bits
    for l in range(N_LAYERS):
        one = LayerStep(CFG, {"x": inp, "params": params[l]})
        one.fwd()
        torch.cuda.synchronize()
        assert np.array_equal(tensor_to_bits(one.y), acts[l]), l
        inp = acts[l]
        del one
    # backward: layer l with the stored input gradient of layer l+1
    d_bits = dy_bits
    for l in range(N_LAYERS - 1, -1, -1):
        one = LayerStep(CFG, {"x": x_bits if l == 0 else acts[l - 1], "params": params[l]})
        one.set_dy_bits(d_bits)
        one.fwd()
        one.bwd()
        torch.cuda.synchronize()
        g_one = one.grads_host()
        g_st = st.layer_grads_host(l)
        for k in g_one:
            assert np.array_equal(g_one[k], g_st[k]), (l, k)
        d_bits = tensor_to_bits(one.dx)
        del one
    assert np.array_equal(d_bits, tensor_to_bits(st.dx))


def test_stack_matches_oracle_and_one_adam_covers_every_layer():
    need_gpu()
    params, x_bits, r_bits = _inputs()
    st = LayerStack(CFG, params, x_bits)
    scale = st.hyper["init_scale"]
    dy_bits = synth.loss_grad_bits(CFG, scale, r_bits)
    st.set_dy_bits(dy_bits)
    st.fwd()
    st.bwd()
    check_device_error()
    out_gpu = host_values(st.y, CFG.dtype)
    dx_gpu = host_values(st.dx, CFG.dtype)
    x = synth.from_bits(x_bits, CFG.dtype).reshape(CFG.tokens, CFG.hidden)
    ps = [{k: synth.from_bits(v, CFG.dtype).reshape(v.shape) for k, v in p.items()} for p in params]
    dout = synth.from_bits(dy_bits, CFG.dtype).reshape(CFG.tokens, CFG.hidden)
    eps = st.hyper["ln_eps"]
    out_o, caches = oracle.stack_fwd(x, ps, CFG.dims(), eps, precision=CFG.dtype)
    dx_o, gr_o = oracle.stack_bwd(caches, ps, CFG.dims(), dout)
    errs = {"out": rel_max_err(out_gpu, out_o), "dx": rel_max_err(dx_gpu, dx_o)}
    for l in range(N_LAYERS):
        g = st.layer_grads_host(l)
        for k in gr_o[l]:
            errs[(l, k)] = rel_max_err(g[k].reshape(gr_o[l][k].shape), gr_o[l][k])
    print({str(k): round(v, 5) for k, v in errs.items()})
    assert all(v <= 2e-2 for v in errs.values()), errs

    # one optimizer call over the L * n_layer_params arena
    hp = st.hyper
    p_in, m_in, v_in = st.master.cpu().numpy(), st.m.cpu().numpy(), st.v.cpu().numpy()
    grad = st.grad.cpu().numpy()
    st.adam()
    torch.cuda.synchronize()
    assert st.scaler()["found_inf"] == 0
    f32 = lambda a: float(np.float32(a))
    pe, _, _, _ = oracle.adam_step(p_in, m_in, v_in, grad, scale, 0, f32(hp["lr"]),
                                   f32(hp["beta1"]), f32(hp["beta2"]), f32(hp["eps"]),
                                   f32(hp["weight_decay"]), CFG.dtype, 0)
    pg = st.master.cpu().numpy()
    lr = f32(hp["lr"])
    assert np.all(np.abs(pg - pe) <= 1e-6 * np.maximum(np.abs(pe), lr))
    n = st.n_layer_params
    for l in range(N_LAYERS):        # every layer's block moved
        blk = slice(l * n, (l + 1) * n)
        assert np.count_nonzero(pg[blk] != p_in[blk]) > 0.9 * np.count_nonzero(grad[blk])


def test_stack_with_gelu_recompute_is_bit_identical():
    """The stack with recompute_gelu (each layer's A written again in its
    backward instead of saved) equals the saving stack bit for bit, and its
    saved workspace is smaller by one A per layer."""
    need_gpu()
    params, x_bits, r_bits = _inputs()
    dy_bits = synth.loss_grad_bits(CFG, synth.HYPER["init_scale"], r_bits)
    runs = []
    for recompute in (False, True):
        st = LayerStack(CFG, params, x_bits, recompute_gelu=recompute)
        st.set_dy_bits(dy_bits)
        st.fwd()
        st.bwd()
        torch.cuda.synchronize()
        check_device_error()
        runs.append((st.acts.clone(), st.dx.clone(), st.grad.clone(), st.saved.numel()))
        del st
    (a0, dx0, g0, s0), (a1, dx1, g1, s1) = runs
    assert torch.equal(a0, a1) and torch.equal(dx0, dx1) and torch.equal(g0, g1)
    assert s0 - s1 >= N_LAYERS * CFG.tokens * CFG.ffn * 2
