"""GPU parity of the tcgen05 GEMM (gptl_gemm) in every operand arrangement
the layer step uses, against the float64 contraction of the same 16-bit
inputs.  The expected value applies the descriptor's documented view rules
(include/gptlayer_parts.h) with numpy; shapes span several tiles and ragged
M/N/K tails."""
import math

import numpy as np
import pytest
import torch

from transformer_layer_step_b200 import gptlayer as G
from gpu_util import need_gpu, dev_tensor, host_values, rounded, stream, check_device_error

pytestmark = pytest.mark.gpu


def _operand_matrix(buf, op, G_idx, ks, rows_needed, k_len):
    """[rows_needed, k_len] float64 matrix the operand contributes for group
    G_idx and k-shard ks; zeros outside the view."""
    x0 = (G_idx % op["x_mod"]) * op["x_mul"] + op["x_off"]
    gdiv = op["g_div"]
    gc = G_idx // gdiv + (ks if op["k_shard"] else 0)
    out = np.zeros((rows_needed, k_len))
    xe, re_, ge = op["x_ext"], op["rows_ext"], op["g_ext"]
    if gc >= ge:
        return out
    plane = buf[gc]                                # [rows_ext, x_ext]
    for r in range(rows_needed):
        for_k = np.arange(k_len)
        if not op["mn_major"]:
            row, xs = r, x0 + for_k
            if row < re_:
                ok = xs < xe
                out[r, ok] = plane[row, xs[ok]]
        else:
            xs, rows = x0 + r, for_k
            if xs < xe:
                ok = rows < re_
                out[r, ok] = plane[rows[ok], xs]
    return out


def _expected(desc, abuf, bbuf):
    M, N, K = desc["M"], desc["N"], desc["K"]
    res = []
    for g in range(desc["groups"]):
        acc = np.zeros((M, N))
        for ks in range(desc["k_shards"]):
            A = _operand_matrix(abuf, desc["a"], g, ks, M, K)
            B = _operand_matrix(bbuf, desc["b"], g, ks, N, K)
            acc += A @ B.T
        res.append(acc)
    return np.stack(res)


def _op(buf_t, x_ext, rows_ext, g_ext, row_pitch, g_pitch, mn, x_mod=1, x_mul=0, x_off=0,
        g_div=None, k_shard=0):
    if g_div is None:
        g_div = 1 if g_ext > 1 else (1 << 30)
    d = dict(x_ext=x_ext, rows_ext=rows_ext, g_ext=g_ext, mn_major=mn, x_mod=x_mod, x_mul=x_mul,
             x_off=x_off, g_div=g_div, k_shard=k_shard)
    c = G.operand(buf_t, x_ext, rows_ext, g_ext, row_pitch, g_pitch, mn, x_mod, x_mul, x_off,
                  g_div, k_shard)
    return d, c


def _run(dtype, M, N, K, groups, k_shards, causal, a_spec, b_spec, out_f32=False, bias=False,
         resid=False, act=G.ACT_NONE, seed=0, std_a=1.0, std_b=0.1, ws_bytes=0, resid_f32=False,
         launches=None, colsum=False, dgelu_out2=False, extras=None):
    """a_spec/b_spec: (shape of the 3-D buffer [g, rows, x], view kwargs).  With
    colsum / dgelu_out2, extras receives the column-sum partials [ceil(M/32)][g][N]
    and the second (GeLU) output of a DGELU epilogue."""
    need_gpu()
    rng = np.random.default_rng(seed)
    abuf = rounded(rng.standard_normal(a_spec[0]) * std_a, dtype)
    bbuf = rounded(rng.standard_normal(b_spec[0]) * std_b, dtype)
    at, bt = dev_tensor(abuf, dtype), dev_tensor(bbuf, dtype)
    ad, ac = _op(at, a_spec[0][2], a_spec[0][1], a_spec[0][0], a_spec[0][2],
                 a_spec[0][1] * a_spec[0][2], **a_spec[1])
    bd, bc = _op(bt, b_spec[0][2], b_spec[0][1], b_spec[0][0], b_spec[0][2],
                 b_spec[0][1] * b_spec[0][2], **b_spec[1])
    desc_py = dict(M=M, N=N, K=K, groups=groups, k_shards=k_shards, causal=causal, a=ad, b=bd)
    exp = _expected(desc_py, abuf, bbuf)
    if out_f32:
        out = torch.full((groups, M, N), float("nan"), dtype=torch.float32, device="cuda")
    else:
        out = torch.zeros((groups, M, N), dtype=torch.float16 if dtype == "fp16" else torch.bfloat16,
                          device="cuda")
    d = G.GemmDesc()
    d.M, d.N, d.K, d.groups, d.k_shards, d.causal = M, N, K, groups, k_shards, causal
    d.a, d.b = ac, bc
    d.out, d.out_f32, d.ldo, d.o_mod, d.o_str_mod, d.o_str_div = out.data_ptr(), int(out_f32), N, 1, 0, M * N
    bias_v = resid_v = aux_v = None
    keep = []
    if bias:
        bias_v = rounded(rng.standard_normal((groups, N)) * 0.5, dtype)
        bt_ = dev_tensor(bias_v, dtype)
        keep.append(bt_)
        d.bias, d.bias_g_stride = bt_.data_ptr(), N
    if resid:
        if resid_f32:
            resid_v = rng.standard_normal((M, N)).astype(np.float32).astype(np.float64)
            rt_ = torch.from_numpy(resid_v.astype(np.float32)).cuda()
            d.resid_f32 = 1
        else:
            resid_v = rounded(rng.standard_normal((M, N)), dtype)
            rt_ = dev_tensor(resid_v, dtype)
        keep.append(rt_)
        d.resid, d.ld_resid = rt_.data_ptr(), N
    if ws_bytes:
        ws = torch.full((ws_bytes // 4,), float("nan"), dtype=torch.float32, device="cuda")
        keep.append(ws)
        d.ws, d.ws_bytes = ws.data_ptr(), ws_bytes
    out2 = None
    if act == G.ACT_GELU or dgelu_out2:
        out2 = torch.zeros_like(out)
        d.out2 = out2.data_ptr()
    cs = None
    if colsum:
        cs = torch.full(((M + 31) // 32, groups, N), float("nan"), dtype=torch.float32, device="cuda")
        d.colsum = cs.data_ptr()
    if act == G.ACT_DGELU:
        aux_v = rounded(rng.standard_normal((groups, M, N)), dtype)
        xt_ = dev_tensor(aux_v, dtype)
        keep.append(xt_)
        d.aux = xt_.data_ptr()
    d.act = act
    n0 = G.launch_count()
    G.gemm(d, dtype, stream())
    check_device_error()
    if launches is not None:
        launches.append(G.launch_count() - n0)
    if extras is not None:
        extras["colsum"] = None if cs is None else cs.cpu().numpy().astype(np.float64)
        extras["out2"] = None if out2 is None or act != G.ACT_DGELU else host_values(out2, dtype)
        extras["aux"] = aux_v
    if bias:
        exp = exp + bias_v[:, None, :]
    if resid:
        exp = exp + resid_v[None]
    if out_f32:
        return exp, out.cpu().numpy(), None
    got = host_values(out, dtype)
    got2 = None
    if act == G.ACT_GELU:
        z = rounded(exp, dtype)
        u = math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)
        exp2 = 0.5 * z * (1 + np.tanh(u))
        got2 = (host_values(out2, dtype), exp2)
    if act == G.ACT_DGELU:
        z = aux_v
        u = math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)
        th = np.tanh(u)
        gp = 0.5 * (1 + th) + 0.5 * z * (1 - th * th) * math.sqrt(2 / math.pi) * (1 + 3 * 0.044715 * z * z)
        exp = exp * gp
    return exp, got, got2


def _close(got, exp, tol, mask=None):
    if mask is not None:
        got, exp = got[mask], exp[mask]
    scale = max(float(np.abs(exp).max()), 1e-6)
    err = float(np.abs(got - exp).max()) / scale
    assert err <= tol, err


DT = ["bf16", "fp16"]


@pytest.mark.parametrize("dtype", DT)
def test_fprop_kmajor_bias_grouped(dtype):
    # column-split style: A shared, B and out grouped; ragged M and K tail
    exp, got, _ = _run(dtype, M=300, N=192, K=160, groups=2, k_shards=1, causal=0,
                       a_spec=((1, 300, 160), dict(mn=0)), b_spec=((2, 192, 160), dict(mn=0)),
                       bias=True)
    _close(got, exp, 8e-3)


@pytest.mark.parametrize("dtype", DT)
def test_fprop_wide_n_resid(dtype):
    exp, got, _ = _run(dtype, M=256, N=640, K=128, groups=1, k_shards=1, causal=0,
                       a_spec=((1, 256, 128), dict(mn=0)), b_spec=((1, 640, 128), dict(mn=0)),
                       bias=True, resid=True)
    _close(got, exp, 8e-3)


@pytest.mark.parametrize("dtype", DT)
def test_bias_gelu_epilogue(dtype):
    exp, got, (got2, exp2) = _run(dtype, M=200, N=256, K=192, groups=2, k_shards=1, causal=0,
                                  a_spec=((1, 200, 192), dict(mn=0)),
                                  b_spec=((2, 256, 192), dict(mn=0)), bias=True, act=G.ACT_GELU)
    _close(got, exp, 8e-3)
    _close(got2, exp2, 1.5e-2)


@pytest.mark.parametrize("dtype", DT)
def test_dgelu_epilogue_mn_major_b(dtype):
    # input-gradient style: B is [g][k][n] (MN-major)
    exp, got, _ = _run(dtype, M=260, N=128, K=256, groups=2, k_shards=1, causal=0,
                       a_spec=((1, 260, 256), dict(mn=0)), b_spec=((2, 256, 128), dict(mn=1)),
                       act=G.ACT_DGELU)
    _close(got, exp, 1e-2)


@pytest.mark.parametrize("dtype", DT)
@pytest.mark.parametrize("M,K,groups", [(260, 256, 2), (700, 512, 3)])
def test_dgelu_colsum_and_recomputed_activation(dtype, M, K, groups):
    """The FFN2 input-gradient GEMM with its two extra epilogue outputs: the
    32-row column sums of the stored dZ (the partials of the FFN1 bias
    gradient; a 32-row group partly past M, and groups wholly past it that
    must not be written) and GeLU of the stored Z again (the activation
    recomputed for the FFN2 weight gradient)."""
    N = 320
    ex = {}
    exp, got, _ = _run(dtype, M=M, N=N, K=K, groups=groups, k_shards=1, causal=0,
                       a_spec=((1, M, K), dict(mn=0)), b_spec=((groups, K, N), dict(mn=1)),
                       act=G.ACT_DGELU, colsum=True, dgelu_out2=True, extras=ex)
    _close(got, exp, 1e-2)
    rows = (M + 31) // 32
    g64 = got.astype(np.float64)
    want = np.stack([g64[:, 32 * r:32 * r + 32, :].sum(axis=1) for r in range(rows)])
    mag = np.stack([np.abs(g64[:, 32 * r:32 * r + 32, :]).sum(axis=1) for r in range(rows)])
    assert ex["colsum"].shape == want.shape
    err = np.abs(ex["colsum"] - want)
    assert np.all(err <= 1e-6 * mag + 1e-30), float(np.max(err / (mag + 1e-30)))
    # GeLU of the stored argument, as the forward's bias-GeLU epilogue computes it
    z = ex["aux"]
    u = math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)
    _close(ex["out2"], 0.5 * z * (1 + np.tanh(u)), 1.5e-2)


@pytest.mark.parametrize("dtype", DT)
def test_recomputed_activation_is_bit_identical(dtype):
    """GeLU recomputed in the DGELU epilogue from a stored Z equals, bit for
    bit, the GeLU that the bias-GeLU epilogue wrote beside that Z."""
    need_gpu()
    M, N, K, groups = 300, 256, 128, 2
    rng = np.random.default_rng(5)
    tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
    at = dev_tensor(rounded(rng.standard_normal((1, M, K)), dtype), dtype)
    bt = dev_tensor(rounded(rng.standard_normal((groups, N, K)) * 0.2, dtype), dtype)
    _, ac = _op(at, K, M, 1, K, M * K, mn=0)
    _, bc = _op(bt, K, N, groups, K, N * K, mn=0)
    z, act1, dz, act2 = (torch.zeros((groups, M, N), dtype=tdt, device="cuda") for _ in range(4))
    d = G.GemmDesc()
    d.M, d.N, d.K, d.groups, d.k_shards, d.causal = M, N, K, groups, 1, 0
    d.a, d.b = ac, bc
    d.out, d.out_f32, d.ldo, d.o_mod, d.o_str_mod, d.o_str_div = z.data_ptr(), 0, N, 1, 0, M * N
    d.out2, d.act = act1.data_ptr(), G.ACT_GELU
    G.gemm(d, dtype, stream())
    d.out, d.out2, d.aux, d.act = dz.data_ptr(), act2.data_ptr(), z.data_ptr(), G.ACT_DGELU
    G.gemm(d, dtype, stream())
    check_device_error()
    assert torch.equal(act1.view(torch.int16), act2.view(torch.int16))


@pytest.mark.parametrize("dtype", DT)
def test_wgrad_both_mn_major_fp32(dtype):
    exp, got, _ = _run(dtype, M=192, N=320, K=384, groups=2, k_shards=1, causal=0,
                       a_spec=((1, 384, 192), dict(mn=1)), b_spec=((2, 384, 320), dict(mn=1)),
                       out_f32=True)
    _close(got, exp, 1e-5)


@pytest.mark.parametrize("dtype", DT)
def test_k_shard_reduction(dtype):
    # row-split style: both operands walk 3 shards along the group axis
    exp, got, _ = _run(dtype, M=384, N=256, K=128, groups=1, k_shards=3, causal=0,
                       a_spec=((3, 384, 128), dict(mn=0, g_div=1 << 30, k_shard=1)),
                       b_spec=((3, 256, 128), dict(mn=0, g_div=1 << 30, k_shard=1)),
                       bias=True, resid=True)
    _close(got, exp, 8e-3)
    # column-split input gradient: B MN-major per shard
    exp, got, _ = _run(dtype, M=256, N=192, K=128, groups=1, k_shards=2, causal=0,
                       a_spec=((2, 256, 128), dict(mn=0, g_div=1 << 30, k_shard=1)),
                       b_spec=((2, 128, 192), dict(mn=1, g_div=1 << 30, k_shard=1)))
    _close(got, exp, 8e-3)


@pytest.mark.parametrize("dtype", DT)
def test_wgrad_split_k(dtype):
    """Few output tiles and a long K: the K loop is split across SMs, the fp32
    partials summed by a second kernel (two launches); deterministic."""
    kw = dict(M=256, N=128, K=8192, groups=1, k_shards=1, causal=0,
              a_spec=((1, 8192, 256), dict(mn=1)), b_spec=((1, 8192, 128), dict(mn=1)),
              out_f32=True, ws_bytes=8 * 256 * 128 * 4)
    nl = []
    exp, got, _ = _run(dtype, launches=nl, **kw)
    _close(got, exp, 5e-5)          # fp32 sums of 8192 products
    assert nl == [2]
    _, got2, _ = _run(dtype, **kw)
    np.testing.assert_array_equal(got, got2)
    # no workspace: one launch, same values up to the summation order
    nl = []
    kw["ws_bytes"] = 0
    _, got3, _ = _run(dtype, launches=nl, **kw)
    assert nl == [1]
    _close(got3, exp, 5e-5)


@pytest.mark.parametrize("dtype", DT)
def test_fp32_out_with_bias_and_fp32_residual(dtype):
    """The residual-stream epilogue: fp32 output of acc + bias (16-bit) +
    residual (16-bit), and a 16-bit output of acc + bias + fp32 residual."""
    kw = dict(M=300, N=256, K=192, groups=1, k_shards=1, causal=0,
              a_spec=((1, 300, 192), dict(mn=0)), b_spec=((1, 256, 192), dict(mn=0)))
    exp, got, _ = _run(dtype, out_f32=True, bias=True, resid=True, **kw)
    _close(got, exp, 1e-5)
    exp, got, _ = _run(dtype, bias=True, resid=True, resid_f32=True, **kw)
    _close(got, exp, 1e-2)


@pytest.mark.parametrize("dtype,out_f32", [("bf16", False), ("fp16", True)])
def test_interleaved_group_output_and_padding(dtype, out_f32):
    """Groups written side by side into a padded buffer (o_mod = 2):
    out + (G % 2) * N + (G / 2) * M * ldo + m * ldo + n, ldo = 2N + 16.  The
    tensor stores are clipped to each group's M x N window, so the 16 padding
    columns of every row keep their sentinel."""
    need_gpu()
    M, N, K, groups = 200, 96, 64, 4
    ldo = 2 * N + 16
    rng = np.random.default_rng(11)
    abuf = rounded(rng.standard_normal((1, M, K)), dtype)
    bbuf = rounded(rng.standard_normal((groups, N, K)) * 0.1, dtype)
    at, bt = dev_tensor(abuf, dtype), dev_tensor(bbuf, dtype)
    _, ac = _op(at, K, M, 1, K, M * K, 0)
    _, bc = _op(bt, K, N, groups, K, N * K, 0)
    tdt = torch.float32 if out_f32 else (torch.float16 if dtype == "fp16" else torch.bfloat16)
    out = torch.full((groups // 2, M, ldo), float("nan"), dtype=tdt, device="cuda")
    d = G.GemmDesc()
    d.M, d.N, d.K, d.groups, d.k_shards, d.causal = M, N, K, groups, 1, 0
    d.a, d.b = ac, bc
    d.out, d.out_f32, d.ldo = out.data_ptr(), int(out_f32), ldo
    d.o_mod, d.o_str_mod, d.o_str_div = 2, N, M * ldo
    G.gemm(d, dtype, stream())
    check_device_error()
    got = out.float().cpu().numpy()
    for g in range(groups):
        exp = abuf[0] @ bbuf[g].T
        part = got[g // 2, :, (g % 2) * N:(g % 2 + 1) * N]
        tol = 1e-5 if out_f32 else 8e-3
        assert float(np.abs(part - exp).max()) <= tol * float(np.abs(exp).max())
    assert np.isnan(got[:, :, 2 * N:]).all()


def _plan(M, N, K, groups, a_spec, b_spec, out_f32=False, ws_bytes=0, dtype="bf16"):
    rng = np.random.default_rng(0)
    at = dev_tensor(rounded(rng.standard_normal(a_spec[0]), dtype), dtype)
    bt = dev_tensor(rounded(rng.standard_normal(b_spec[0]), dtype), dtype)
    _, ac = _op(at, a_spec[0][2], a_spec[0][1], a_spec[0][0], a_spec[0][2],
                a_spec[0][1] * a_spec[0][2], **a_spec[1])
    _, bc = _op(bt, b_spec[0][2], b_spec[0][1], b_spec[0][0], b_spec[0][2],
                b_spec[0][1] * b_spec[0][2], **b_spec[1])
    out = torch.empty((groups, M, N), dtype=torch.float32 if out_f32 else torch.bfloat16, device="cuda")
    ws = torch.empty((max(ws_bytes, 16) // 4,), dtype=torch.float32, device="cuda")
    d = G.GemmDesc()
    d.M, d.N, d.K, d.groups, d.k_shards, d.causal = M, N, K, groups, 1, 0
    d.a, d.b = ac, bc
    d.out, d.out_f32, d.ldo, d.o_mod, d.o_str_div = out.data_ptr(), int(out_f32), N, 1, M * N
    if ws_bytes:
        d.ws, d.ws_bytes = ws.data_ptr(), ws_bytes
    return G.gemm_plan(d, dtype)


def test_pipeline_modes_with_several_tiles_per_sm():
    """Each way of using an SM's two MMA pipelines (tiles alternating between
    them, both on one tile's K halves, 256-row tiles split by M) on shapes
    with more tiles than SMs, so that every CTA walks several tiles (in the
    banded tile order); the library reports which way it chose
    (gptl_gemm_plan) and the cases must cover all three."""
    need_gpu()
    cases = [
        # the attention-input projection's shape: 256-row tiles, ~2 per SM
        dict(dtype="bf16", M=8192, N=2304, K=768, groups=1, k_shards=1, causal=0,
             a_spec=((1, 8192, 768), dict(mn=0)), b_spec=((1, 2304, 768), dict(mn=0)), bias=True),
        # MN-major operands, fp32 output, ragged M and N tails, three groups
        dict(dtype="fp16", M=1000, N=1024, K=2048, groups=3, k_shards=1, causal=0,
             a_spec=((3, 2048, 1000), dict(mn=1)), b_spec=((1, 2048, 1024), dict(mn=1)), out_f32=True),
        # one 128-row tile per group, many groups: tiles alternate
        dict(dtype="fp16", M=128, N=256, K=64, groups=400, k_shards=1, causal=0,
             a_spec=((1, 128, 64), dict(mn=0)), b_spec=((400, 256, 64), dict(mn=0))),
        # few tiles, long K, no workspace: K halves
        dict(dtype="bf16", M=256, N=256, K=4096, groups=1, k_shards=1, causal=0,
             a_spec=((1, 256, 4096), dict(mn=0)), b_spec=((1, 256, 4096), dict(mn=0)), out_f32=True),
        # weight-gradient shape with a workspace: split-K slices as well
        dict(dtype="bf16", M=768, N=1024, K=8192, groups=1, k_shards=1, causal=0,
             a_spec=((1, 8192, 768), dict(mn=1)), b_spec=((1, 8192, 1024), dict(mn=1)),
             out_f32=True, ws_bytes=8 * 768 * 1024 * 4),
    ]
    modes = set()
    for kw in cases:
        bn, split, mode = _plan(kw["M"], kw["N"], kw["K"], kw["groups"], kw["a_spec"], kw["b_spec"],
                                kw.get("out_f32", False), kw.get("ws_bytes", 0), kw["dtype"])
        modes.add(mode)
        exp, got, _ = _run(**kw)
        tol = 5e-5 if kw.get("out_f32") else 8e-3
        _close(got, exp, tol)
        # the same plan twice gives the same bits
        _, got2, _ = _run(**kw)
        np.testing.assert_array_equal(got, got2)
    assert modes == {G.GEMM_ALTERNATE, G.GEMM_K_HALVES, G.GEMM_M256}, modes
