"""The overflow check folded into the backward (gpt_layer_bwd_checked +
adam_step_fp32_master_prechecked, "Megatron-LM overview" §3.1 dynamic loss
scaling) against the scanning path (gpt_layer_bwd + adam_step_fp32_master,
whose overflow pass re-reads the whole gradient arena).

* Decisions, bit for bit: on the same seeded step with a clean dOut, with
  one NaN, one +inf, and a row of dOut so large that fp32 weight gradients
  overflow, the flag the checked backward sets equals the scan of the arena
  it wrote (gptl_check_overflow), and is 0 exactly when the arena is finite.
* Results, bit for bit: two steps through either path leave the same
  output, input gradient, gradients, master weights, moments, 16-bit
  weights and scaler state.
"""
import numpy as np
import pytest
import torch

from transformer_layer_step_b200 import gptlayer as G
from transformer_layer_step_b200 import synth
from transformer_layer_step_b200.harness import LayerStep, bits_to_tensor
from gpu_util import need_gpu, check_device_error

pytestmark = pytest.mark.gpu

CFGS = [synth.LayerConfig("ck-bf16-t2", 2, 256, 256, 4, 1024, 2, synth.BF16),
        synth.LayerConfig("ck-fp16-t4", 1, 128, 512, 8, 2048, 4, synth.FP16)]


def _step(cfg, inp, dy_bits):
    ls = LayerStep(cfg, inp)
    ls.set_dy_bits(dy_bits)
    return ls


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
@pytest.mark.parametrize("poison", ["clean", "nan", "inf", "huge_row"])
def test_checked_flag_equals_the_scan(cfg, poison):
    need_gpu()
    inp = synth.make_inputs(cfg, seed=3, variant="biased", with_r=True)
    dy = synth.loss_grad_bits(cfg, 1024.0, inp["r"]).copy()
    big = 65504.0 if cfg.dtype == synth.FP16 else 3.0e38
    if poison == "nan":
        dy[5, 7] = synth.to_bits(np.array([np.nan]), cfg.dtype)[0]
    elif poison == "inf":
        dy[9, 3] = synth.to_bits(np.array([np.inf]), cfg.dtype)[0]
    elif poison == "huge_row":
        dy[:, 11] = synth.to_bits(np.full(cfg.tokens, big), cfg.dtype)
    ls = _step(cfg, inp, dy)
    ls.fwd()
    ls.state[2] = 7                          # found_inf: the checked backward must reset it
    ls.bwd(checked=True)
    torch.cuda.synchronize()
    flag = int(ls.state[2].item())
    scan_state = ls.state.clone()
    G.check_overflow(ls.n_params, ls.grad, scan_state, ls.stream())
    torch.cuda.synchronize()
    check_device_error()
    scan = int(scan_state[2].item())
    finite = bool(torch.isfinite(ls.grad).all().item())
    assert flag == scan == (0 if finite else 1), (flag, scan, finite)
    if poison in ("nan", "inf"):
        assert flag == 1
    if poison == "clean":
        assert flag == 0


@pytest.mark.parametrize("cfg", CFGS, ids=lambda c: c.name)
def test_checked_step_matches_the_scanning_step(cfg):
    need_gpu()
    inp = synth.make_inputs(cfg, seed=4, variant="biased", with_r=True)
    dy = synth.loss_grad_bits(cfg, synth.HYPER["init_scale"], inp["r"])
    a, b = _step(cfg, inp, dy), _step(cfg, inp, dy)
    for _ in range(2):
        a.step()
        b.step(fused_check=True)
    torch.cuda.synchronize()
    check_device_error()
    for name in ("y", "dx", "grad", "master", "m", "v", "w16", "state"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    assert a.scaler()["step"] == 2
