"""Forward and backward of one pre-LayerNorm GPT layer with Megatron tensor
parallelism, computed shard by shard in float64.  Test infrastructure only.

Layout of the parameters (shard-major, t shards):
  ln1_g, ln1_b, ln2_g, ln2_b  [h]             replicated
  w_qkv  [t, 3h/t, h]   b_qkv [t, 3h/t]       column split: shard i owns the
                                              Q, K, V rows of heads
                                              i*a/t .. (i+1)*a/t - 1
  w_o    [t, h, h/t]    b_o   [h]             row split (input columns)
  w_1    [t, f/t, h]    b_1   [t, f/t]        column split
  w_2    [t, h, f/t]    b_2   [h]             row split
Activations are [T, h] with token row r = j*s + p (batch j, position p).

Column split: each shard computes its own output columns from the full
input; row split: each shard multiplies its slice of the input and the
partial products are summed ("Megatron-LM 3D parallelism", §1; "Megatron-LM
overview", §2.2).  Here the sum is an explicit float64 loop over shards.

Precision.  With precision=None every value is exact float64.  With
precision="fp16" or "bf16" the layer is computed the way the pages' mixed
precision defines it ("Megatron-LM overview", §3.1: FP16 matrix math; the
layer computes in fp16/bf16): every activation tensor that one step of the
path hands to the next is held in the 16-bit type (round to nearest, ties to
even), while the arithmetic inside a step stays exact.  The stored tensors
are, forward: L1, C = [Q|K|V], P (the fused attention keeps the scores on
chip; its probabilities are 16-bit as a matrix operand), O, L2, Z,
A = gelu(Z); backward: dZ (the GeLU backward is applied to dOut W2 before
the store, as the fused bias-GeLU's backward), dL2, dO, dV, dS, dQ, dK, dL1,
and the 16-bit copy of dH that the out-projection's backward GEMMs read.
The softmax backward's row term sum_q P_pq dP_pq is formed as dO_p . O_p
(equal in exact arithmetic, since O = P V) from the stored dO and O; the
exact mode uses the plain sum.  The residual stream H = X + attention and its gradient dH are the
FP32 side of mixed precision (like the master weights, they are never
matrix operands): they stay exact here.  The layer outputs Out and dX are
returned unrounded (their own store is the caller's last rounding) and the
weight and bias gradients are fp32 quantities, returned exactly.
"""
from __future__ import annotations

import math
import numpy as np

from .optim import round_to_16

# Plainest readings where the pages are silent:
#   LayerNorm: affine, biased variance over h, eps passed in (1e-5 by default).
#   GeLU: the tanh form used by GPT-2 / Megatron's fused bias-GeLU.
#   Softmax: scores scaled by 1/sqrt(d) before the causal mask; masked
#            entries are excluded, so their probability is exactly 0.
GELU_C = math.sqrt(2.0 / math.pi)
GELU_A = 0.044715


def layer_norm_fwd(x: np.ndarray, g: np.ndarray, b: np.ndarray, eps: float):
    """Row-wise LayerNorm. Returns (y, mu, rstd, xhat)."""
    mu = x.mean(axis=1)
    xc = x - mu[:, None]
    var = (xc * xc).mean(axis=1)
    rstd = 1.0 / np.sqrt(var + eps)
    xhat = xc * rstd[:, None]
    return xhat * g[None, :] + b[None, :], mu, rstd, xhat


def layer_norm_bwd(gy: np.ndarray, xhat: np.ndarray, rstd: np.ndarray, g: np.ndarray):
    """Backward of y = g*xhat + b.  Returns (dx, dg, db)."""
    dg = (gy * xhat).sum(axis=0)
    db = gy.sum(axis=0)
    gh = gy * g[None, :]
    dx = rstd[:, None] * (gh - gh.mean(axis=1, keepdims=True)
                          - xhat * (gh * xhat).mean(axis=1, keepdims=True))
    return dx, dg, db


def gelu(z: np.ndarray) -> np.ndarray:
    u = GELU_C * (z + GELU_A * z ** 3)
    return 0.5 * z * (1.0 + np.tanh(u))


def gelu_prime(z: np.ndarray) -> np.ndarray:
    u = GELU_C * (z + GELU_A * z ** 3)
    th = np.tanh(u)
    return 0.5 * (1.0 + th) + 0.5 * z * (1.0 - th * th) * GELU_C * (1.0 + 3.0 * GELU_A * z * z)


def causal_softmax(z: np.ndarray) -> np.ndarray:
    """Row softmax over q <= p of an [s, s] score block (already scaled);
    entries with q > p get probability exactly 0."""
    s = z.shape[0]
    p = np.zeros_like(z)
    for r in range(s):
        row = z[r, : r + 1]
        e = np.exp(row - row.max())
        p[r, : r + 1] = e / e.sum()
    return p


def attention_head_fwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, precision=None, noise=None,
                       noise_at=None):
    """One (batch, head) block of causal self-attention: returns (P, O).
    With a 16-bit precision P is a stored (rounded) value; O is returned
    unrounded (the layer stores it)."""
    d = q.shape[1]
    z = (q @ k.T) / math.sqrt(d)
    p = _store(causal_softmax(z), precision, noise, "p", noise_at)
    return p, p @ v


def attention_head_bwd(q: np.ndarray, k: np.ndarray, v: np.ndarray, p: np.ndarray,
                       do: np.ndarray, o: np.ndarray, precision=None, noise=None, noise_at=None):
    """Backward of one (batch, head) block of causal self-attention, given
    its probabilities P (as attention_head_fwd returns them), the output
    gradient dO and the output O.  Returns (dQ, dK, dV).

    dP = dO V^T; dV = P^T dO; dZ = P (dP - r) with the row term
    r_p = sum_q P_pq dP_pq; dS = dZ / sqrt(d); dQ = dS K; dK = dS^T Q.  In
    the mixed-precision mode dV, dS (the operand of both products), dQ and dK
    are stored, and the row term is formed as dO_p . O_p from the stored dO
    and O (equal in exact arithmetic, since O = P V); dP stays exact, as the
    fused kernel keeps it on chip."""
    st = lambda a, name: _store(a, precision, noise, name, noise_at)
    d = q.shape[1]
    dp = do @ v.T
    dv = st(p.T @ do, "dv")
    if precision is None:
        rowterm = (p * dp).sum(axis=1, keepdims=True)
    else:
        rowterm = (do * o).sum(axis=1, keepdims=True)
    dsc = st((p * (dp - rowterm)) * (1.0 / math.sqrt(d)), "ds")
    return st(dsc @ k, "dq"), st(dsc.T @ q, "dk"), dv


# The tensors the mixed-precision mode holds in the 16-bit type, by name, in
# the order the step produces them (see the module doc).
FWD_STORE_POINTS = ("l1", "c", "p", "o", "l2", "z", "act")
BWD_STORE_POINTS = ("dz", "dl2", "dh16", "do", "dv", "ds", "dq", "dk", "dl1")
STORE_POINTS = FWD_STORE_POINTS + BWD_STORE_POINTS


def _store(a: np.ndarray, precision, noise=None, name=None, noise_at=None):
    """An activation tensor as the next step reads it (see the module doc).
    `noise`, when given, is applied to the value just before it is rounded:
    a callable that returns the value times (1 + a small relative error),
    standing for the rounding of a fp32-accumulating implementation, so that
    a test can measure how far two correct implementations of the 16-bit
    method drift apart.  `noise_at`, a set of store-point names, limits the
    noise to those stores (None: every store)."""
    assert name in STORE_POINTS, name
    if precision is None:
        return a
    if noise is not None and (noise_at is None or name in noise_at):
        a = noise(a)
    return round_to_16(a, precision)


def _check(dims, params):
    b, s, h, a, f, t = (dims[k] for k in "bshaft")
    assert h % a == 0 and a % t == 0 and f % t == 0
    assert params["w_qkv"].shape == (t, 3 * h // t, h)
    assert params["w_o"].shape == (t, h, h // t)
    assert params["w_1"].shape == (t, f // t, h)
    assert params["w_2"].shape == (t, h, f // t)
    return b, s, h, a, f, t


def layer_fwd(x: np.ndarray, params: dict, dims: dict, eps: float = 1e-5, precision=None,
              noise=None, noise_at=None):
    """Forward pass.  x: [T, h] float64.  precision: None (exact) or the
    16-bit type the activations are stored in; noise, noise_at: see _store
    (both are kept in the cache for the backward pass).
    Returns (out, cache)."""
    st = lambda a, name: _store(a, precision, noise, name, noise_at)
    if noise_at is not None:
        assert set(noise_at) <= set(STORE_POINTS), noise_at
    b, s, h, a, f, t = _check(dims, params)
    d = h // a
    hs, a_s = h // t, a // t            # hidden columns and heads per shard
    T = b * s
    assert x.shape == (T, h)

    # 1. LN1
    l1, mu1, rstd1, xhat1 = layer_norm_fwd(x, params["ln1_g"], params["ln1_b"], eps)
    l1 = st(l1, "l1")

    # 2. QKV column-split GEMM: C_i = L1 W_qkv,i^T + b_qkv,i  -> [Q_i | K_i | V_i]
    c = st(np.stack([l1 @ params["w_qkv"][i].T + params["b_qkv"][i][None, :] for i in range(t)]), "c")

    # 3. causal attention, head by head; head eta of shard i is global head i*a/t+eta
    probs = np.zeros((t, b, a_s, s, s))
    o = np.zeros((t, T, hs))
    for i in range(t):
        for j in range(b):
            rows = slice(j * s, (j + 1) * s)
            for eta in range(a_s):
                cols = slice(eta * d, (eta + 1) * d)
                qh = c[i, rows, 0 * hs:1 * hs][:, cols]
                kh = c[i, rows, 1 * hs:2 * hs][:, cols]
                vh = c[i, rows, 2 * hs:3 * hs][:, cols]
                pr, oh = attention_head_fwd(qh, kh, vh, precision, noise, noise_at)
                probs[i, j, eta] = pr
                o[i, rows, cols] = st(oh, "o")

    # 4. out-projection, row split: partial products summed over shards, bias
    #    added once after the sum, then the residual
    y_attn = np.zeros((T, h))
    for i in range(t):
        y_attn += o[i] @ params["w_o"][i].T
    hid = x + y_attn + params["b_o"][None, :]

    # 5. LN2
    l2, mu2, rstd2, xhat2 = layer_norm_fwd(hid, params["ln2_g"], params["ln2_b"], eps)
    l2 = st(l2, "l2")

    # 6. FFN1 column split with fused bias + GeLU
    z = st(np.stack([l2 @ params["w_1"][i].T + params["b_1"][i][None, :] for i in range(t)]), "z")
    act = st(gelu(z), "act")

    # 7. FFN2 row split: shard sum, bias, residual
    y_mlp = np.zeros((T, h))
    for i in range(t):
        y_mlp += act[i] @ params["w_2"][i].T
    out = hid + y_mlp + params["b_2"][None, :]

    cache = dict(x=x, l1=l1, mu1=mu1, rstd1=rstd1, xhat1=xhat1, c=c, probs=probs, o=o,
                 hid=hid, l2=l2, mu2=mu2, rstd2=rstd2, xhat2=xhat2, z=z, act=act,
                 precision=precision, noise=noise, noise_at=noise_at)
    return out, cache


def layer_bwd(cache: dict, params: dict, dims: dict, dout: np.ndarray, keep: dict = None):
    """Backward pass given dOut (already multiplied by the loss scale).
    Returns (dx, grads) with grads in the same shard-major layout as params.
    When `keep` is a dict, the backward's intermediate tensors are left in it
    (dz, dl2, dh, dh16, do, dc, dl1), so that a test can check each stored
    tensor against its step recomputed from the stored inputs."""
    b, s, h, a, f, t = _check(dims, params)
    d = h // a
    hs, a_s = h // t, a // t
    T = b * s
    precision, noise, noise_at = cache.get("precision"), cache.get("noise"), cache.get("noise_at")
    st = lambda a, name: _store(a, precision, noise, name, noise_at)
    gr = {}

    # FFN2 (row split): each shard's weight gradient and input gradient
    gr["b_2"] = dout.sum(axis=0)
    gr["w_2"] = np.stack([dout.T @ cache["act"][i] for i in range(t)])
    d_act = np.stack([dout @ params["w_2"][i] for i in range(t)])

    # GeLU backward and FFN1 (column split); the input gradient is the sum
    # of the shards' partial products
    dz = st(d_act * gelu_prime(cache["z"]), "dz")
    gr["b_1"] = dz.sum(axis=1)
    gr["w_1"] = np.stack([dz[i].T @ cache["l2"] for i in range(t)])
    dl2 = np.zeros((T, h))
    for i in range(t):
        dl2 += dz[i] @ params["w_1"][i]
    dl2 = st(dl2, "dl2")

    # LN2 backward plus the residual path
    dln, gr["ln2_g"], gr["ln2_b"] = layer_norm_bwd(dl2, cache["xhat2"], cache["rstd2"],
                                                   params["ln2_g"])
    dhid = dout + dln
    dhid16 = st(dhid, "dh16")           # the matrix operand copy of dH

    # out-projection (row split)
    gr["b_o"] = dhid.sum(axis=0)
    gr["w_o"] = np.stack([dhid16.T @ cache["o"][i] for i in range(t)])
    do = st(np.stack([dhid16 @ params["w_o"][i] for i in range(t)]), "do")

    # attention backward, head by head
    c = cache["c"]
    dc = np.zeros_like(c)
    for i in range(t):
        for j in range(b):
            rows = slice(j * s, (j + 1) * s)
            for eta in range(a_s):
                cols = slice(eta * d, (eta + 1) * d)
                qh = c[i, rows, 0 * hs:1 * hs][:, cols]
                kh = c[i, rows, 1 * hs:2 * hs][:, cols]
                vh = c[i, rows, 2 * hs:3 * hs][:, cols]
                pr = cache["probs"][i, j, eta]
                doh = do[i, rows, cols]
                dq, dk, dv = attention_head_bwd(qh, kh, vh, pr, doh, cache["o"][i, rows, cols],
                                                precision, noise, noise_at)
                dc[i, rows, 0 * hs:1 * hs][:, cols] = dq
                dc[i, rows, 1 * hs:2 * hs][:, cols] = dk
                dc[i, rows, 2 * hs:3 * hs][:, cols] = dv

    # QKV (column split): per-shard weight and bias grads, shard-summed dL1
    gr["b_qkv"] = dc.sum(axis=1)
    gr["w_qkv"] = np.stack([dc[i].T @ cache["l1"] for i in range(t)])
    dl1 = np.zeros((T, h))
    for i in range(t):
        dl1 += dc[i] @ params["w_qkv"][i]
    dl1 = st(dl1, "dl1")

    # LN1 backward plus the residual path
    dln1, gr["ln1_g"], gr["ln1_b"] = layer_norm_bwd(dl1, cache["xhat1"], cache["rstd1"],
                                                    params["ln1_g"])
    dx = dhid + dln1
    if keep is not None:
        keep.update(dz=dz, dl2=dl2, dh=dhid, dh16=dhid16, do=do, dc=dc, dl1=dl1)
    return dx, gr


def stack_fwd(x: np.ndarray, params_list: list, dims: dict, eps: float = 1e-5, precision=None):
    """Forward of a stack of layers of one shape ("Training GPT-2 with
    Megatron-LM" §4.1 runs --num-layers 32 of them): layer l's output is
    layer l+1's input.  With a precision, the output a layer hands to the
    next is held in the 16-bit type, the store between the two layers.
    Returns (out, caches); out is the last layer's output, unrounded."""
    caches = []
    h = x
    for l, p in enumerate(params_list):
        if l > 0 and precision is not None:
            h = round_to_16(h, precision)
        h, c = layer_fwd(h, p, dims, eps, precision)
        caches.append(c)
    return h, caches


def stack_bwd(caches: list, params_list: list, dims: dict, dout: np.ndarray):
    """Backward through stack_fwd's layers in reverse order: layer l's dX is
    layer l-1's dOut, held in the 16-bit type between the two layers under a
    precision.  Returns (dx, grads) with grads[l] the gradients of layer l."""
    grads = [None] * len(params_list)
    d = dout
    last = len(params_list) - 1
    for l in range(last, -1, -1):
        prec = caches[l].get("precision")
        if l < last and prec is not None:
            d = round_to_16(d, prec)
        d, grads[l] = layer_bwd(caches[l], params_list[l], dims, d)
    return d, grads
