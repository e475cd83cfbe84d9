"""The transposed weight copies written by the optimizer step
(gpt_layer_adam_step, gpt_layer_transpose_weights, gptl_weights' *_t
fields): the input-gradient products of the backward read the weights with
the reduction index contiguous, and the optimizer step, which writes the
16-bit weights anyway, writes those transposed copies too, instead of the
backward transposing the weights again every step.

* The copies are exact: every shard of the four weight matrices, transposed.
* Results, bit for bit: steps through the copying path (one layer and a
  stack of layers, with the scanning and the folded overflow check) leave
  the same output, input gradient, gradients, master weights, moments,
  16-bit weights and scaler state as the plain path; a skipped step leaves
  the copies untouched.
"""
import numpy as np
import pytest
import torch

from transformer_layer_step_b200 import gptlayer as G
from transformer_layer_step_b200 import synth
from transformer_layer_step_b200.harness import LayerStack, LayerStep
from gpu_util import need_gpu, check_device_error

pytestmark = pytest.mark.gpu

CFGS = [synth.LayerConfig("wt-bf16-t2", 2, 256, 256, 4, 1024, 2, synth.BF16),
        synth.LayerConfig("wt-fp16-t4-d80", 1, 128, 640, 8, 2560, 4, synth.FP16)]

MATS = (("w_qkv", lambda c: (3 * c.hidden // c.tp, c.hidden)), ("w_o", lambda c: (c.hidden, c.hidden // c.tp)),
        ("w_1", lambda c: (c.ffn // c.tp, c.hidden)), ("w_2", lambda c: (c.hidden, c.ffn // c.tp)))


def _assert_copies(ls, cfg, layers=1):
    """w16t holds every shard of each weight matrix transposed, at w16's offsets."""
    names = dict(zip(G.PARAM_NAMES, ls.offsets))
    per = ls.n_params // layers
    w = ls.w16.view(torch.int16)
    wt = ls.w16t.view(torch.int16)
    for l in range(layers):
        for name, shape in MATS:
            rows, cols = shape(cfg)
            off = l * per + names[name]
            n = cfg.tp * rows * cols
            a = w[off:off + n].view(cfg.tp, rows, cols)
            b = wt[off:off + n].view(cfg.tp, cols, rows)
            assert torch.equal(a.transpose(1, 2), b), (l, name)


def _run(ls, dy_bits, steps, fused_check):
    ls.set_dy_bits(dy_bits)
    for _ in range(steps):
        ls.step(fused_check=fused_check)
    torch.cuda.synchronize()
    check_device_error()
    return {k: getattr(ls, k).clone() for k in ("y", "dx", "grad", "master", "m", "v", "w16", "state")}


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
@pytest.mark.parametrize("fused_check", [False, True])
def test_layer_steps_with_weight_copies_are_bit_identical(cfg, fused_check):
    need_gpu()
    inp = synth.make_inputs(cfg, seed=4, variant="biased", with_r=True)
    dy = synth.loss_grad_bits(cfg, 1024.0, inp["r"])
    plain = _run(LayerStep(cfg, inp), dy, 3, fused_check)
    ls = LayerStep(cfg, inp, weight_copies=True)
    torch.cuda.synchronize()
    _assert_copies(ls, cfg)                  # the first copies
    copied = _run(ls, dy, 3, fused_check)
    for k in plain:
        assert torch.equal(plain[k], copied[k]), k
    _assert_copies(ls, cfg)                  # kept up to date by every step


def test_skipped_step_leaves_the_copies():
    need_gpu()
    cfg = CFGS[0]
    inp = synth.make_inputs(cfg, seed=5, variant="biased", with_r=True)
    dy = synth.loss_grad_bits(cfg, 1024.0, inp["r"]).copy()
    dy[3, 5] = synth.to_bits(np.array([np.inf]), cfg.dtype)[0]
    ls = LayerStep(cfg, inp, weight_copies=True)
    ls.set_dy_bits(dy)
    before = (ls.w16t.clone(), ls.w16.clone(), ls.master.clone())
    ls.step(fused_check=True)
    torch.cuda.synchronize()
    check_device_error()
    assert ls.scaler()["found_inf"] == 1
    assert torch.equal(before[0], ls.w16t) and torch.equal(before[1], ls.w16)
    assert torch.equal(before[2], ls.master)


def test_stack_with_weight_copies_is_bit_identical():
    need_gpu()
    cfg = synth.CONFIGS["tiny"]
    layers = [synth.make_inputs(cfg, seed=20 + l, variant="biased")["params"] for l in range(3)]
    first = synth.make_inputs(cfg, seed=6, variant="biased", with_r=True)
    dy = synth.loss_grad_bits(cfg, 1024.0, first["r"])
    out = []
    for copies in (False, True):
        st = LayerStack(cfg, layers, first["x"], weight_copies=copies)
        st.set_dy_bits(dy)
        for _ in range(2):
            st.step()
        torch.cuda.synchronize()
        check_device_error()
        out.append({k: getattr(st, k).clone() for k in ("acts", "dx", "grad", "master", "w16")})
        if copies:
            _assert_copies(st, cfg, layers=3)
        del st
    for k in out[0]:
        assert torch.equal(out[0][k], out[1][k]), k
