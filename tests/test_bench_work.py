"""The algorithmic work that bench.py divides by measured time for its
roofline figures, counted here another way.

* FLOPs: the twelve linear products of one step enumerated one by one with
  their sharded shapes (forward, input gradient, weight gradient; two FLOPs
  per multiply-add), and the causal attention products counted by brute
  force over the lower triangle q <= p of small heads.
* Bytes: the optimizer's per-parameter traffic from the arrays it reads and
  writes, and the transposed weight copies from the parameter layout that
  the library reports (the matrix entries of the arena).
"""
import itertools

import pytest

import bench
from transformer_layer_step_b200 import gptlayer as G
from transformer_layer_step_b200 import synth


def _linear_products(c):
    """(name, M, N, K, groups) of every linear product of one step: M rows
    of the output, N columns, reduction length K, one product per shard."""
    T, h, f, t = c.tokens, c.hidden, c.ffn, c.tp
    fwd = [("qkv", T, 3 * h // t, h), ("outproj", T, h, h // t),
           ("ffn1", T, f // t, h), ("ffn2", T, h, f // t)]
    out = []
    for name, M, N, K in fwd:
        out.append((name, M, N, K, t))
        out.append((name + " input grad", M, K, N, t))     # dX = dY W: [M, K] over N
        out.append((name + " weight grad", N, K, M, t))    # dW = dY^T X: [N, K] over M
    return out


@pytest.mark.parametrize("name", list(synth.CONFIGS))
def test_linear_flops_match_the_enumerated_products(name):
    c = synth.CONFIGS[name]
    prods = _linear_products(c)
    assert len(prods) == 12
    total = sum(2 * M * N * K * g for _, M, N, K, g in prods)
    assert bench.step_flops(c)["linear"] == total


def _causal_pair_count(s):
    return sum(1 for q, p in itertools.product(range(s), range(s)) if q <= p)


@pytest.mark.parametrize("b,s,h,a", [(1, 1, 64, 1), (2, 7, 128, 2), (3, 13, 192, 3)])
def test_attention_flops_count_the_lower_triangle(b, s, h, a):
    cfg = synth.LayerConfig("t", b, s, h, a, 4 * h, 1, synth.FP16)
    d = h // a
    pairs = _causal_pair_count(s)
    assert pairs == s * (s + 1) // 2
    # forward: S = Q K^T and O = P V, one d-long dot product per (q, p) pair
    fwd = b * a * 2 * (2 * d * pairs)
    # backward: dP = dO V^T, dV = P^T dO, dQ = dS K, dK = dS^T Q
    bwd = b * a * 4 * (2 * d * pairs)
    fl = bench.step_flops(cfg)
    assert fl["attn_fwd"] == fwd
    assert fl["attn_bwd"] == bwd
    assert fl["causal"] == fl["linear"] + 3 * fwd


@pytest.mark.parametrize("name", ["tiny", "gpt2-117m", "large-h10240"])
def test_optimizer_bytes_per_parameter_and_copies(name):
    c = synth.CONFIGS[name]
    sh = G.make_shape(c.batch, c.seq, c.hidden, c.heads, c.ffn, c.tp, c.dtype)
    offs, n = G.param_layout(sh)
    per = dict(zip(G.PARAM_NAMES, offs))
    # reads: master, m, v, gradient (fp32); writes: master, m, v (fp32), 16-bit weights
    per_param = 4 * 4 + 3 * 4 + 2
    nb = bench.kernel_bytes(c, n)
    assert nb["O2 adam"] == per_param * n
    assert nb["O1 overflow"] == 4 * n
    # the four weight matrices' entries: every shard's [rows][cols], each
    # matrix filling its span of the arena up to the next tensor (its bias)
    # but for the alignment padding (offsets are multiples of 64)
    h, f, t = c.hidden, c.ffn, c.tp
    shards = {"w_qkv": (3 * h // t, h), "w_o": (h, h // t), "w_1": (f // t, h), "w_2": (h, f // t)}
    names = list(G.PARAM_NAMES)
    mats = 0
    for w, (rows, cols) in shards.items():
        entries = t * rows * cols
        span = offs[names.index(w) + 1] - per[w]
        assert 0 <= span - entries < 64, w
        mats += entries
    nbc = bench.kernel_bytes(c, n, weight_copies=True)
    assert nbc["O2 adam"] - nb["O2 adam"] == 2 * mats
    # with the copies the backward has no weight transposes to do; without,
    # it reads and writes every matrix entry once
    assert nb["B0 weights^T"] == 4 * mats


def test_roofline_arithmetic_on_recorded_launches():
    """The per-kernel summary and the roofline figures from a made-up launch
    record of two steps at the hidden-10240 shapes: achieved = algorithmic
    work / summed launch time, frac = achieved / peak (the sustained GEMM
    rate for the tensor-core families), shares over the step's total."""
    c = synth.CONFIGS["large-h10240"]
    sh = G.make_shape(c.batch, c.seq, c.hidden, c.heads, c.ffn, c.tp, c.dtype)
    _, n = G.param_layout(sh)
    peaks = {"hbm_gbs": 5000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1000.0}
    flops = bench.step_flops(c)
    K = 2
    one_step = [("gemm", "F2 qkv", 1.0), ("gemm", "F10 ffn2", 3.0),
                ("attn_fwd", "F3-F5 attn", 2.0), ("adam", "O2 adam", 4.0)]
    rows, kinds, ms_step = bench.summarize_kernels(one_step * K, K, c, n, peaks, flops)
    assert ms_step == pytest.approx(10.0)
    assert kinds["gemm"]["ms_per_step"] == pytest.approx(4.0)
    assert kinds["gemm"]["launches_per_step"] == 2
    assert kinds["adam"]["share"] == pytest.approx(0.4)
    adam = next(r for r in rows if r["step"] == "O2 adam")
    want_gbs = 30 * n / 4.0e-3 / 1e9
    assert adam["GB/s"] == pytest.approx(want_gbs, rel=1e-3)
    assert adam["frac_hbm"] == pytest.approx(want_gbs / 5000.0, abs=1e-3)
    roof = bench.kernel_rooflines(kinds, rows, c, n, flops, peaks, "test")
    want_tf = flops["linear"] / 4.0e-3 / 1e12
    assert roof["gemm"]["achieved"] == pytest.approx(want_tf, rel=1e-3)
    assert roof["gemm"]["frac"] == pytest.approx(want_tf / 1000.0, rel=1e-3)
    assert roof["attn_fwd"]["achieved"] == pytest.approx(flops["attn_fwd"] / 2.0e-3 / 1e12, rel=1e-3)
    assert roof["adam"]["bytes"] == 30 * n
    assert roof["adam"]["achieved"] == pytest.approx(want_gbs, rel=1e-3)
