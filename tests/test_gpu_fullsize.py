"""The two largest workloads at their full sizes.

* Full layer parity, forward and backward, element by element: the 2.4B
  model's layer ("Training GPT-2 with Megatron-LM" §4.1: hidden 2560, 32
  heads of 80, ffn 10240, seq 2048, tp 4, fp16) at one sequence per step,
  and the hidden-10240 layer ("Megatron-LM 3D parallelism", the 128-GPU
  example: 80 heads of 128, ffn 40960, seq 2048, tp 4, bf16).  Out, dX and
  all 12 gradients against the oracle with the bars of test_gpu_layer.py
  (fp16 also against the all-float64 oracle).  At these sizes the GEMMs run
  their largest tilings (K up to 40960 over four shards, 256-row tiles, the
  weight gradients' long token reductions) and the attention backward its
  2048-long rows with head_dim 80 and 128.
* Sampled forward rows of the 2.4B layer at its full batch of four: the
  causal mask makes the first positions of a sequence self-contained
  (their attention never looks further), and LayerNorm and the MLP act row
  by row, so the oracle run on the first 64 positions of a sequence alone
  gives exactly those rows of the full layer's output.  The last sequence
  of the batch is compared with the 2e-2 * RMS bar.
* The skip/backoff path of dynamic loss scaling at the hidden-10240 layer:
  one +inf written into a shard of dW1 after the backward must skip the
  step bit-exactly (master, m, v and the 16-bit weights untouched, step
  count unchanged) and halve the scale; the next clean step goes through,
  and sampled chunks of its Adam update match the oracle within the
  spec bar (1e-6 relative).
"""
import dataclasses
import functools

import numpy as np
import pytest
import torch

import oracle
from transformer_layer_step_b200 import gptlayer as G
from transformer_layer_step_b200 import synth
from transformer_layer_step_b200.harness import LayerStep
from gpu_util import need_gpu, host_values, check_device_error, rel_max_err
from layer_parity import run_gpu, check_against_oracle

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

PREFIX = 64
FULL = {
    "gpt-2.4b-b1": dataclasses.replace(synth.CONFIGS["gpt-2.4b"], name="gpt-2.4b-b1", batch=1),
    "large-h10240": synth.CONFIGS["large-h10240"],
}


@functools.lru_cache(maxsize=2)
def _inputs(name):
    cfg = FULL[name] if name in FULL else synth.CONFIGS[name]
    return synth.make_inputs(cfg, seed=0, variant="biased", with_r=True)


@pytest.mark.parametrize("name", list(FULL))
def test_full_size_layer_parity(name):
    need_gpu()
    cfg = FULL[name]
    inp = _inputs(name)
    dy_bits = synth.loss_grad_bits(cfg, synth.HYPER["init_scale"], inp["r"])
    out_gpu, dx_gpu, grads_gpu = run_gpu(cfg, inp, dy_bits)
    check_against_oracle(cfg, inp, dy_bits, out_gpu, dx_gpu, grads_gpu, eps=synth.HYPER["ln_eps"],
                         exact=cfg.dtype == synth.FP16)


def test_sampled_forward_rows_full_batch():
    need_gpu()
    cfg = synth.CONFIGS["gpt-2.4b"]
    inp = synth.make_inputs(cfg, seed=0, variant="biased", with_r=False)
    ls = LayerStep(cfg, inp)
    ls.fwd()
    check_device_error()
    eps = ls.hyper["ln_eps"]
    p = {k: synth.from_bits(v, cfg.dtype).reshape(v.shape) for k, v in inp["params"].items()}
    x_bits = inp["x"].reshape(cfg.tokens, cfg.hidden)
    sub = dataclasses.replace(cfg, batch=1, seq=PREFIX)
    j = cfg.batch - 1
    rows = slice(j * cfg.seq, j * cfg.seq + PREFIX)
    x = synth.from_bits(x_bits[rows], cfg.dtype).reshape(PREFIX, cfg.hidden)
    out_o, _ = oracle.layer_fwd(x, p, sub.dims(), eps, precision=cfg.dtype)
    got = host_values(ls.y[rows], cfg.dtype)
    err = rel_max_err(got, out_o)
    print(cfg.name, "sequence", j, "rows 0..63: max|gpu - oracle| / rms =", round(err, 5))
    assert err <= 2e-2


def test_injected_overflow_skips_and_backs_off_large():
    need_gpu()
    cfg = synth.CONFIGS["large-h10240"]
    inp = _inputs("large-h10240")
    ls = LayerStep(cfg, inp)
    hp = ls.hyper
    ls.set_dy_bits(synth.loss_grad_bits(cfg, hp["init_scale"], inp["r"]))
    ls.fwd()
    ls.bwd()
    torch.cuda.synchronize()
    # +inf into dW1 of shard 2 at a seeded index
    w1_off = ls.offsets[G.PARAM_NAMES.index("w_1")]
    shard = (cfg.ffn // cfg.tp) * cfg.hidden
    idx = w1_off + 2 * shard + int(np.random.default_rng(2).integers(shard))
    ls.grad[idx] = float("inf")
    before = [t.clone() for t in (ls.master, ls.m, ls.v, ls.w16)]
    ls.adam()
    ls.scale_update()
    torch.cuda.synchronize()
    st = ls.scaler()
    assert st["found_inf"] == 1
    assert st["scale"] == hp["init_scale"] * hp["backoff_factor"]
    assert st["growth_tracker"] == 0 and st["step"] == 0
    for a, b in zip(before, (ls.master, ls.m, ls.v, ls.w16)):
        assert torch.equal(a, b)
    del before
    # a clean step at the backed-off scale
    ls.set_dy_bits(synth.loss_grad_bits(cfg, st["scale"], inp["r"]))
    ls.fwd()
    ls.bwd()
    torch.cuda.synchronize()
    n = ls.n_params
    rng = np.random.default_rng(5)
    starts = [int(s) for s in rng.integers(0, n - (1 << 20), 3)] + [w1_off + 2 * shard]
    chunks = [slice(s0, s0 + (1 << 20)) for s0 in starts]
    saved = [(ls.master[c].cpu().numpy(), ls.m[c].cpu().numpy(), ls.v[c].cpu().numpy(),
              ls.grad[c].cpu().numpy()) for c in chunks]
    ls.adam()
    ls.scale_update()
    torch.cuda.synchronize()
    check_device_error()
    st2 = ls.scaler()
    assert st2["found_inf"] == 0 and st2["step"] == 1 and st2["growth_tracker"] == 1
    assert st2["scale"] == st["scale"]
    f32 = lambda x: float(np.float32(x))
    lr = f32(hp["lr"])
    for c, (p_in, m_in, v_in, g_in) in zip(chunks, saved):
        assert oracle.found_inf(g_in) == 0
        pe, me, ve, _ = oracle.adam_step(p_in, m_in, v_in, g_in, st["scale"], 0, lr,
                                         f32(hp["beta1"]), f32(hp["beta2"]), f32(hp["eps"]),
                                         f32(hp["weight_decay"]), cfg.dtype, 0)
        pg, mg, vg = ls.master[c].cpu().numpy(), ls.m[c].cpu().numpy(), ls.v[c].cpu().numpy()
        assert np.all(np.abs(pg - pe) <= 1e-6 * np.maximum(np.abs(pe), lr))
        assert np.all(np.abs(vg - ve) <= 1e-6 * np.abs(ve) + 1e-45)
        assert np.all(np.abs(mg - me) <= 1e-6 * np.maximum(np.abs(me), np.sqrt(np.mean(me ** 2))))
