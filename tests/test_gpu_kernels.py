"""GPU parity of the bandwidth kernels against the CPU oracle: LayerNorm
forward/backward, column sums, overflow check, fused Adam, loss-scale
update, clipping and accumulation."""
import dataclasses
import math

import numpy as np
import pytest
import torch

import oracle
from transformer_layer_step_b200 import gptlayer as G
from transformer_layer_step_b200 import synth
from transformer_layer_step_b200.harness import LayerStep
from gpu_util import (need_gpu, dev_tensor, host_values, rounded, stream, check_device_error,
                      rel_max_err)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype,rows,h", [("bf16", 333, 768), ("fp16", 130, 128),
                                          ("fp16", 97, 1024), ("bf16", 70, 2560),
                                          ("bf16", 9, 10240)])
def test_layernorm_fwd_bwd(dtype, rows, h):
    need_gpu()
    rng = np.random.default_rng(rows + h)
    x = rounded(rng.standard_normal((rows, h)) * 2 + 0.5, dtype)
    g = rounded(1 + 0.1 * rng.standard_normal(h), dtype)
    b = rounded(0.1 * rng.standard_normal(h), dtype)
    gy = rounded(rng.standard_normal((rows, h)), dtype)
    res = rounded(rng.standard_normal((rows, h)), dtype)
    xt, gt, bt, gyt, rt = (dev_tensor(a, dtype) for a in (x, g, b, gy, res))
    y = torch.empty_like(xt)
    mu = torch.empty(rows, dtype=torch.float32, device="cuda")
    rstd = torch.empty_like(mu)
    G.layernorm_fwd(rows, h, dtype, xt, gt, bt, 1e-5, y, mu, rstd, stream())
    ye, mue, rse, xhat = oracle.layer_norm_fwd(x, g, b, 1e-5)
    torch.cuda.synchronize()
    assert rel_max_err(host_values(y, dtype), ye) < 2e-2
    np.testing.assert_allclose(mu.cpu().numpy(), mue, rtol=0, atol=1e-5)
    np.testing.assert_allclose(rstd.cpu().numpy(), rse, rtol=1e-5)

    dx = torch.empty_like(xt)
    dg = torch.empty(h, dtype=torch.float32, device="cuda")
    db = torch.empty_like(dg)
    dsum = torch.empty_like(dg)
    scratch = torch.empty(G.layernorm_bwd_scratch_bytes(rows, h), dtype=torch.uint8, device="cuda")
    G.layernorm_bwd(rows, h, dtype, gyt, xt, mu, rstd, gt, rt, dx, dg, db, dsum, scratch, stream())
    check_device_error()
    dxe, dge, dbe = oracle.layer_norm_bwd(gy, xhat, rse, g)
    dxe = dxe + res
    assert rel_max_err(host_values(dx, dtype), dxe) < 2e-2
    assert rel_max_err(dg.cpu().numpy(), dge) < 2e-3
    assert rel_max_err(db.cpu().numpy(), dbe) < 1e-4
    assert rel_max_err(dsum.cpu().numpy(), host_values(dx, dtype).sum(axis=0)) < 1e-4


@pytest.mark.parametrize("dtype,rows,n,groups", [("bf16", 8192, 768, 1), ("fp16", 130, 256, 2),
                                                 ("fp16", 1000, 1920, 4)])
def test_colsum(dtype, rows, n, groups):
    need_gpu()
    rng = np.random.default_rng(n)
    a = rounded(rng.standard_normal((groups, rows, n)), dtype)
    at = dev_tensor(a, dtype)
    out = torch.empty(groups * n, dtype=torch.float32, device="cuda")
    scratch = torch.empty(G.colsum_scratch_bytes(n, groups), dtype=torch.uint8, device="cuda")
    G.colsum(rows, n, groups, n, rows * n, dtype, at, out, scratch, stream())
    check_device_error()
    np.testing.assert_allclose(out.cpu().numpy(), a.sum(axis=1).reshape(-1), rtol=0, atol=1e-3)


def test_overflow_and_scaler_decisions():
    need_gpu()
    n = 1 << 20
    g = torch.from_numpy(synth.random_fp32(n, 1)).cuda()
    state = torch.zeros(8, dtype=torch.int32, device="cuda")
    for pos, bad in [(None, None), (0, math.inf), (n - 1, -math.inf), (123457, math.nan),
                     (n // 2, math.inf)]:
        gg = g.clone()
        if pos is not None:
            gg[pos] = bad
        state[2] = 7
        G.check_overflow(n, gg, state, stream())
        torch.cuda.synchronize()
        assert int(state[2]) == oracle.found_inf(gg.cpu().numpy())


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_adam_matches_oracle(dtype):
    need_gpu()
    cfg = dataclasses.replace(synth.CONFIGS["tiny"], dtype=dtype)
    ls = LayerStep(cfg, synth.make_inputs(cfg))
    n = ls.n_params
    rng = np.random.default_rng(3)
    hp = ls.hyper
    master = ls.master.cpu().numpy().astype(np.float64)
    m = np.zeros(n)
    v = np.zeros(n)
    state = dict(scale=hp["init_scale"], growth_tracker=0, step=0)
    for step in range(4):
        grad = (rng.standard_normal(n) * 1e-3 * state["scale"]).astype(np.float32)
        if step == 2:
            grad[n // 3] = np.inf                       # this step must be skipped
        ls.grad.copy_(torch.from_numpy(grad))
        m_in, v_in, p_in = ls.m.cpu().numpy(), ls.v.cpu().numpy(), ls.master.cpu().numpy()
        w_in = ls.w16.clone()
        ls.adam()
        ls.scale_update()
        torch.cuda.synchronize()
        f = oracle.found_inf(grad)
        f32 = lambda x: float(np.float32(x))
        pe, me, ve, we = oracle.adam_step(p_in, m_in, v_in, grad, state["scale"], state["step"],
                                          f32(hp["lr"]), f32(hp["beta1"]), f32(hp["beta2"]),
                                          f32(hp["eps"]), f32(hp["weight_decay"]), dtype, f)
        state = oracle.loss_scale_update(state, f, hp["growth_interval"], hp["growth_factor"],
                                         hp["backoff_factor"], hp["min_scale"])
        sc = ls.scaler()
        assert sc["found_inf"] == f
        assert (sc["scale"], sc["growth_tracker"], sc["step"]) == \
            (state["scale"], state["growth_tracker"], state["step"])
        pg, mg, vg = ls.master.cpu().numpy(), ls.m.cpu().numpy(), ls.v.cpu().numpy()
        if f:
            assert np.array_equal(pg, p_in) and np.array_equal(mg, m_in) and np.array_equal(vg, v_in)
            assert torch.equal(ls.w16, w_in)
            continue
        lr = f32(hp["lr"])
        assert np.all(np.abs(pg - pe) <= 1e-6 * np.maximum(np.abs(pe), lr))
        assert np.all(np.abs(vg - ve) <= 1e-6 * np.abs(ve) + 1e-45)
        assert np.all(np.abs(mg - me) <= 1e-6 * np.maximum(np.abs(me), np.sqrt(np.mean(me ** 2))))
        # the 16-bit copy is the RNE cast of the GPU's own fp32 master
        wg = ls.w16.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(wg, oracle.cast_to_16(pg.astype(np.float64), dtype))


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
def test_clipped_adam_matches_oracle(dtype):
    """adam_step_fp32_master_clip against the oracle's global-norm clip and
    Adam: the reported norm and coefficient, the update, the skip on
    overflow; unclipped steps bit-equal to adam_step_fp32_master; the norm
    bit-reproducible."""
    need_gpu()
    cfg = dataclasses.replace(synth.CONFIGS["tiny"], dtype=dtype)
    ls = LayerStep(cfg, synth.make_inputs(cfg))
    n = ls.n_params
    rng = np.random.default_rng(4)
    hp = ls.hyper
    f32 = lambda x: float(np.float32(x))
    max_norm = 1.0
    ws = torch.zeros(G.CLIP_WORKSPACE_BYTES // 4, dtype=torch.float32, device="cuda")
    state = dict(scale=hp["init_scale"], growth_tracker=0, step=0)
    # target norms of the unscaled gradient: below, far above, overflow, just
    # below and just above the threshold
    for step, target in enumerate([0.3, 5.0, None, 0.9999, 1.0001, 40.0]):
        S = state["scale"]
        grad = rng.standard_normal(n)
        grad = (grad / np.sqrt((grad ** 2).sum()) * (target or 1.0) * S).astype(np.float32)
        if target is None:
            grad[n // 5] = np.inf
        ls.grad.copy_(torch.from_numpy(grad))
        m_in, v_in, p_in = ls.m.cpu().numpy(), ls.v.cpu().numpy(), ls.master.cpu().numpy()
        w_in = ls.w16.clone()
        plain = [ls.master.clone(), ls.m.clone(), ls.v.clone(), ls.w16.clone(), ls.state.clone()]
        G.adam_step_clip(n, ls.master, ls.m, ls.v, ls.grad, ls.w16, dtype, hp["lr"], hp["beta1"],
                         hp["beta2"], hp["eps"], hp["weight_decay"], max_norm, ws, ls.state,
                         stream())
        torch.cuda.synchronize()
        norm_got, coef_got = float(ws[0]), float(ws[1])
        if step == 0:            # the same inputs again: bit-identical norm
            ws2 = torch.zeros_like(ws)
            again = [t.clone() for t in plain]
            G.adam_step_clip(n, again[0], again[1], again[2], ls.grad, again[3], dtype, hp["lr"],
                             hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], max_norm,
                             ws2, again[4], stream())
            torch.cuda.synchronize()
            assert torch.equal(ws2[:2], ws[:2])
        check_device_error()
        f = oracle.found_inf(grad)
        assert ls.scaler()["found_inf"] == f
        ls.scale_update()
        torch.cuda.synchronize()
        pe, me, ve, _ = (p_in, m_in, v_in, None)
        if not f:
            norm_ref = oracle.grad_norm(grad, S)
            coef_ref = oracle.clip_coefficient(norm_ref, max_norm)
            assert abs(norm_got - norm_ref) <= 1e-6 * norm_ref, (norm_got, norm_ref)
            assert (coef_got == 1.0) == (coef_ref == 1.0), (coef_got, coef_ref)
            assert abs(coef_got - coef_ref) <= 1e-6 * coef_ref
            assert (coef_ref < 1.0) == (target > max_norm)
            pe, me, ve, _ = oracle.adam_step(p_in, m_in, v_in, grad, S, state["step"], f32(hp["lr"]),
                                             f32(hp["beta1"]), f32(hp["beta2"]), f32(hp["eps"]),
                                             f32(hp["weight_decay"]), dtype, f, clip_coef=coef_ref)
        state = oracle.loss_scale_update(state, f, hp["growth_interval"], hp["growth_factor"],
                                         hp["backoff_factor"], hp["min_scale"])
        sc = ls.scaler()
        assert (sc["scale"], sc["growth_tracker"], sc["step"]) == \
            (state["scale"], state["growth_tracker"], state["step"])
        pg, mg, vg = ls.master.cpu().numpy(), ls.m.cpu().numpy(), ls.v.cpu().numpy()
        if f:
            assert np.array_equal(pg, p_in) and np.array_equal(mg, m_in) and np.array_equal(vg, v_in)
            assert torch.equal(ls.w16, w_in)
            continue
        lr = f32(hp["lr"])
        assert np.all(np.abs(pg - pe) <= 1e-6 * np.maximum(np.abs(pe), lr))
        assert np.all(np.abs(vg - ve) <= 1e-6 * np.abs(ve) + 1e-45)
        assert np.all(np.abs(mg - me) <= 1e-6 * np.maximum(np.abs(me), np.sqrt(np.mean(me ** 2))))
        wg = ls.w16.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(wg, oracle.cast_to_16(pg.astype(np.float64), dtype))
        if coef_got == 1.0:      # no clipping: the plain optimizer step, bit for bit
            G.adam_step(n, plain[0], plain[1], plain[2], ls.grad, plain[3], dtype, hp["lr"],
                        hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], plain[4], stream())
            torch.cuda.synchronize()
            assert torch.equal(plain[0], ls.master) and torch.equal(plain[1], ls.m)
            assert torch.equal(plain[2], ls.v) and torch.equal(plain[3], ls.w16)


def test_grad_accumulate_is_fp32_addition():
    need_gpu()
    rng = np.random.default_rng(12)
    n = (1 << 20) + 4 * 37
    parts = []
    for _ in range(3):
        g = (rng.standard_normal(n) * 10.0 ** rng.integers(-12, 12, n)).astype(np.float32)
        parts.append(g)
    parts[1][:100] = -parts[0][:100]                          # exact cancellation
    parts[1][100:200] = parts[0][100:200] * np.float32(2.0 ** -24)   # addends near half an ulp
    acc_t = torch.from_numpy(parts[0].copy()).cuda()
    want = parts[0]
    for g in parts[1:]:
        G.grad_accumulate(n, acc_t, torch.from_numpy(g).cuda(), stream())
        want = oracle.accumulate(want, g)
    check_device_error()
    got = acc_t.cpu().numpy()
    np.testing.assert_array_equal(got.view(np.uint32), want.view(np.uint32))
