"""The layer-parity check shared by the GPU layer tests: run one layer step
through the C ABI, then compare Out, dX and the 12 gradients with the
oracle (the bars are described in test_gpu_layer.py)."""
import numpy as np
import pytest
import torch

import oracle
from transformer_layer_step_b200 import synth
from transformer_layer_step_b200.harness import LayerStep
from gpu_util import host_values, check_device_error, rel_max_err

TOL = 2e-2
# relative size of the fp32-like rounding noise in the drift measurement
DRIFT = 2.0 ** -22


def _errs(out_gpu, dx_gpu, grads_gpu, out_o, dx_o, gr_o, stat=rel_max_err):
    errs = {"out": stat(out_gpu, out_o), "dx": stat(dx_gpu, dx_o)}
    for k in gr_o:
        errs[k] = stat(grads_gpu[k].reshape(gr_o[k].shape), gr_o[k])
    return errs


def rel_rms_err(got, ref):
    return float(np.sqrt(np.mean((got - ref) ** 2)) / max(np.sqrt(np.mean(ref ** 2)), 1e-30))


def run_gpu(cfg, inp, dy_bits):
    ls = LayerStep(cfg, inp)
    ls.set_dy_bits(dy_bits)
    ls.fwd()
    ls.bwd()
    check_device_error()
    out = host_values(ls.y, cfg.dtype)
    dx = host_values(ls.dx, cfg.dtype)
    grads = ls.grads_host()
    del ls
    torch.cuda.empty_cache()
    return out, dx, grads


def check_against_oracle(cfg, inp, dy_bits, out_gpu, dx_gpu, grads_gpu, eps=1e-5, exact=True):
    """Asserts the bars of test_gpu_layer.py; returns the distances."""
    x = synth.from_bits(inp["x"], cfg.dtype).reshape(cfg.tokens, cfg.hidden)
    p = {k: synth.from_bits(v, cfg.dtype).reshape(v.shape) for k, v in inp["params"].items()}
    dout = synth.from_bits(dy_bits, cfg.dtype).reshape(cfg.tokens, cfg.hidden)
    r5 = lambda d: {k: round(v, 5) for k, v in d.items()}
    vs_exact = {}
    if exact:
        out_e, cache = oracle.layer_fwd(x, p, cfg.dims(), eps)
        dx_e, gr_e = oracle.layer_bwd(cache, p, cfg.dims(), dout)
        del cache
        vs_exact = _errs(out_gpu, dx_gpu, grads_gpu, out_e, dx_e, gr_e)
        del out_e, dx_e, gr_e
    out_o, cache = oracle.layer_fwd(x, p, cfg.dims(), eps, precision=cfg.dtype)
    dx_o, gr_o = oracle.layer_bwd(cache, p, cfg.dims(), dout)
    del cache
    errs = _errs(out_gpu, dx_gpu, grads_gpu, out_o, dx_o, gr_o)
    rms_errs = _errs(out_gpu, dx_gpu, grads_gpu, out_o, dx_o, gr_o, stat=rel_rms_err)
    bad = {("rms", k): v for k, v in rms_errs.items() if not v <= TOL}
    if cfg.dtype == synth.FP16:
        bad.update({k: v for k, v in errs.items() if not v <= TOL})
        if exact:
            bad.update({("float64", k): v for k, v in vs_exact.items() if not v <= TOL})
    over = {k: v for k, v in errs.items() if not v <= TOL} if cfg.dtype == synth.BF16 else {}
    floor = {}
    if over:
        # the drift of bf16 storage on this very step: the method again, with
        # fp32-sized noise before each 16-bit store, against the method
        rng = np.random.default_rng(1)
        noise = lambda a: a * (1.0 + DRIFT * rng.standard_normal(a.shape))
        out_n, cache = oracle.layer_fwd(x, p, cfg.dims(), eps, precision=cfg.dtype, noise=noise)
        dx_n, gr_n = oracle.layer_bwd(cache, p, cfg.dims(), dout)
        del cache
        # Out and dX of the GPU are 16-bit tensors: the other implementation
        # stores them too (the gradients are fp32 on both sides)
        floor = _errs(synth.from_bits(synth.to_bits(out_n, cfg.dtype), cfg.dtype).reshape(out_n.shape),
                      synth.from_bits(synth.to_bits(dx_n, cfg.dtype), cfg.dtype).reshape(dx_n.shape),
                      gr_n, out_o, dx_o, gr_o)
        bad.update({("defect", k): (v, floor[k]) for k, v in over.items() if not v <= 2.0 * floor[k]})
    print(cfg.name, {"vs_method": r5(errs), "rms_err": r5(rms_errs), "vs_float64": r5(vs_exact),
                     "drift_floor": r5(floor)})
    assert not bad, (bad, errs)
    if over:
        pytest.xfail(f"measured bf16 limit: max-abs / RMS {r5(over)} above {TOL}, each within "
                     f"twice the drift of bf16 storage on this step {r5({k: floor[k] for k in over})}; "
                     f"RMS errors {r5({k: rms_errs[k] for k in over})}; every other bar met")
    return errs
