"""GPU parity of the whole layer step (gpt_layer_fwd, gpt_layer_bwd through
the C ABI) against the float64 oracle on the same seeded inputs.

Bar: for Out, dX and each of the 12 gradients,
max|gpu - oracle| <= 2e-2 * RMS(oracle), the oracle run at the method's own
precision (activations handed between steps held in the 16-bit type; see
oracle/layer.py).  The gradients are those of the scaled loss (the criterion
is scale-invariant).  Every tensor also meets an RMS-error bar of 2e-2, and
every fp16 tensor meets the 2e-2 max-abs bar against the all-float64 oracle
(the plain definition) as well.

One measured limit stands, for bf16 only.  bf16 keeps 8 significant bits,
and two correct implementations of the bf16 method that differ only in how
their fp32 sums round drift apart by more than 2e-2 * RMS in max-abs on
heavy-tailed tensors (tests/test_oracle_precision.py,
test_bf16_drift_floor_exceeds_the_bar_on_w_qkv): the QKV weight gradient,
whose largest entries are about ten times its RMS, and at the hidden-10240
shape a few more.  When a bf16 tensor misses the max-abs bar, the test
measures that drift on the same step (the oracle again with 2^-22 relative
noise before each 16-bit store) and reports an expected failure with both
numbers if the GPU stays within twice it and every other bar holds; beyond
twice the drift it fails.  It is never passed on a wider bar."""
import pytest
import torch

from transformer_layer_step_b200 import synth
from transformer_layer_step_b200.harness import LayerStep
from gpu_util import need_gpu, check_device_error
from layer_parity import run_gpu, check_against_oracle

pytestmark = pytest.mark.gpu

SMALL = {
    # several tiles in every GEMM, ragged tails, t = 2 and t = 4
    "small-bf16-t2": synth.LayerConfig("small-bf16-t2", 2, 256, 256, 4, 1024, 2, synth.BF16),
    "small-fp16-t4-d80": synth.LayerConfig("small-fp16-t4-d80", 1, 384, 640, 8, 2560, 4, synth.FP16),
    "small-bf16-d128": synth.LayerConfig("small-bf16-d128", 3, 128, 512, 4, 2048, 1, synth.BF16),
}


def _run_and_compare(cfg, variant, with_r, seed=0):
    need_gpu()
    inp = synth.make_inputs(cfg, seed=seed, variant=variant, with_r=with_r)
    dy_bits = synth.loss_grad_bits(cfg, synth.HYPER["init_scale"], inp["r"] if with_r else None)
    out_gpu, dx_gpu, grads_gpu = run_gpu(cfg, inp, dy_bits)
    return check_against_oracle(cfg, inp, dy_bits, out_gpu, dx_gpu, grads_gpu,
                                eps=synth.HYPER["ln_eps"])


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("variant,with_r", [("biased", True), ("plain", False)])
def test_small_layers(name, variant, with_r):
    _run_and_compare(SMALL[name], variant, with_r)


@pytest.mark.parametrize("variant,with_r", [("plain", False), ("biased", True)])
def test_tiny_config(variant, with_r):
    _run_and_compare(synth.CONFIGS["tiny"], variant, with_r)


@pytest.mark.parametrize("name", ["gpt2-117m", "gpt2-345m"])
def test_full_size_configs(name):
    _run_and_compare(synth.CONFIGS[name], "biased", True)


def test_repeat_is_bitwise_deterministic():
    need_gpu()
    cfg = SMALL["small-bf16-t2"]
    inp = synth.make_inputs(cfg, variant="biased", with_r=True)
    ls = LayerStep(cfg, inp)
    ls.set_dy_bits(synth.loss_grad_bits(cfg, 1024.0, inp["r"]))
    ls.fwd(); ls.bwd()
    y1, dx1, g1 = ls.y.clone(), ls.dx.clone(), ls.grad.clone()
    ls.fwd(); ls.bwd()
    torch.cuda.synchronize()
    assert torch.equal(y1, ls.y) and torch.equal(dx1, ls.dx) and torch.equal(g1, ls.grad)


def test_cuda_graph_of_the_step_matches_eager_launches():
    """The whole step (fwd, bwd, overflow check, Adam, scale update) captured
    as one CUDA graph and replayed gives bit-identical outputs, gradients,
    weights and scaler state to launching it kernel by kernel (the library
    makes no host synchronisation or allocation inside a step)."""
    need_gpu()
    cfg = synth.CONFIGS["gpt2-117m"]
    inp = synth.make_inputs(cfg, variant="biased", with_r=True)

    def fresh():
        ls = LayerStep(cfg, inp)
        ls.set_dy_bits(synth.loss_grad_bits(cfg, ls.hyper["init_scale"], inp["r"]))
        return ls

    eager = fresh()
    for _ in range(2):
        eager.step()
    torch.cuda.synchronize()

    graphed = fresh()
    graphed.step()                          # eager first step: shared-memory opt-ins are set
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        graphed.step()                      # captured, not run
    g.replay()
    torch.cuda.synchronize()
    check_device_error()
    for name in ("y", "dx", "grad", "master", "m", "v", "w16", "state"):
        assert torch.equal(getattr(eager, name), getattr(graphed, name)), name


@pytest.mark.parametrize("name", ["small-bf16-t2", "small-fp16-t4-d80"])
def test_gelu_recompute_is_bit_identical(name):
    """Selective recompute of the FFN activation (the shape's recompute_gelu):
    A = GeLU(Z) is not saved but written again from the saved Z by the FFN2
    input-gradient GEMM.  Output, input gradient and every gradient equal the
    saving run's bit for bit, and the saved workspace is smaller by A."""
    need_gpu()
    cfg = SMALL[name]
    inp = synth.make_inputs(cfg, variant="biased", with_r=True)
    dy = synth.loss_grad_bits(cfg, synth.HYPER["init_scale"], inp["r"])
    runs = []
    for recompute in (False, True):
        ls = LayerStep(cfg, inp, recompute_gelu=recompute)
        ls.set_dy_bits(dy)
        ls.fwd()
        ls.scratch.fill_(0xFF)               # the backward may not rely on scratch contents
        ls.bwd()
        torch.cuda.synchronize()
        check_device_error()
        runs.append((ls.y.clone(), ls.dx.clone(), ls.grad.clone(), ls.saved.numel()))
        del ls
    (y0, dx0, g0, s0), (y1, dx1, g1, s1) = runs
    assert torch.equal(y0, y1) and torch.equal(dx0, dx1) and torch.equal(g0, g1)
    assert s0 - s1 >= cfg.tokens * cfg.ffn * 2
