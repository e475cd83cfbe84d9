"""Seeded synthetic inputs for one GPT layer training step.

This module only draws random numbers, rounds them to the 16-bit storage
type and arranges them in the tensor-parallel shard-major layout.  It holds
none of the layer's arithmetic: both the CUDA path and the CPU oracle receive
the arrays it returns, and neither imports the other.

Workloads (the GPT shapes the Megatron-LM pages train):
  * tiny          hidden 128, 4 heads, ffn 512, seq 64, batch 2, tp 2, fp16
  * gpt2-117m     hidden 768, 12 heads, ffn 3072, seq 1024, batch 8, tp 1, bf16
                  (GPT-2 117M layer shape, "Training GPT-2 with Megatron-LM",
                  §3 learning-rate table)
  * gpt2-345m     hidden 1024, 16 heads, ffn 4096, seq 1024, batch 8, tp 4, fp16
                  (same table; "4096-wide FFN split into 4 blocks", §1)
  * gpt-2.4b      hidden 2560, 32 heads, ffn 10240, seq 2048, batch 4, tp 4,
                  fp16 ("Training GPT-2 with Megatron-LM", §4.1 2.4B recipe)
  * large-h10240  hidden 10240, 80 heads, ffn 40960, seq 2048, batch 1, tp 4,
                  bf16, weight std 0.006 ("Megatron-LM 3D parallelism",
                  §4 128-GPU example)

Draw order (numpy PCG64, one generator per call): X, W_qkv, W_o, W_1, W_2,
then for the "biased" variant b_qkv, b_o, b_1, b_2, gamma1-1, beta1,
gamma2-1, beta2, and last R (the loss weights).  Linear weights are drawn
unsharded in [out, in] orientation and then split into shards.
"""
from __future__ import annotations

import dataclasses
import numpy as np

FP16 = "fp16"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    name: str
    batch: int
    seq: int
    hidden: int
    heads: int
    ffn: int
    tp: int
    dtype: str
    w_std: float = 0.02

    @property
    def tokens(self) -> int:
        return self.batch * self.seq

    @property
    def head_dim(self) -> int:
        return self.hidden // self.heads

    def dims(self) -> dict:
        return dict(b=self.batch, s=self.seq, h=self.hidden, a=self.heads,
                    f=self.ffn, t=self.tp)


CONFIGS = {
    c.name: c for c in [
        LayerConfig("tiny", 2, 64, 128, 4, 512, 2, FP16),
        LayerConfig("gpt2-117m", 8, 1024, 768, 12, 3072, 1, BF16),
        LayerConfig("gpt2-345m", 8, 1024, 1024, 16, 4096, 4, FP16),
        LayerConfig("gpt-2.4b", 4, 2048, 2560, 32, 10240, 4, FP16),
        LayerConfig("large-h10240", 1, 2048, 10240, 80, 40960, 4, BF16, 0.006),
    ]
}

# Optimizer and scaler hyper-parameters shared by every workload.
HYPER = dict(lr=6e-5, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.0,
             init_scale=65536.0, growth_interval=1000, growth_factor=2.0,
             backoff_factor=0.5, min_scale=1.0, ln_eps=1e-5)

PARAM_NAMES = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
               "ln2_g", "ln2_b", "w_1", "b_1", "w_2", "b_2")


# --------------------------------------------------------------------------
# 16-bit storage rounding (input preparation only)
# --------------------------------------------------------------------------
def to_bits(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round-to-nearest-even into fp16 or bf16; returns the uint16 bit pattern."""
    if dtype == FP16:
        return np.asarray(x, dtype=np.float64).astype(np.float16).view(np.uint16)
    if dtype == BF16:
        f = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
        u = f.view(np.uint32).astype(np.uint64)
        nan = np.isnan(f)
        # add 0x7FFF plus the lowest kept bit, then drop the low 16 bits
        rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
        out = rounded.astype(np.uint16)
        out[nan] = 0x7FC0
        return out
    raise ValueError(dtype)


def from_bits(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of a uint16 fp16/bf16 bit pattern."""
    bits = np.ascontiguousarray(bits, dtype=np.uint16)
    if dtype == FP16:
        return bits.view(np.float16).astype(np.float64)
    if dtype == BF16:
        return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    raise ValueError(dtype)


# --------------------------------------------------------------------------
# Tensor-parallel layout (which rows/columns each shard owns)
# --------------------------------------------------------------------------
def shard_qkv_rows(w: np.ndarray, t: int) -> np.ndarray:
    """[3h, ...] (rows Q(all heads); K; V) -> [t, 3h/t, ...] with shard i
    holding [Q_i; K_i; V_i], Q_i being the rows of heads i*a/t .. (i+1)*a/t-1."""
    three_h = w.shape[0]
    h = three_h // 3
    parts = []
    for i in range(t):
        sl = slice(i * h // t, (i + 1) * h // t)
        parts.append(np.concatenate([w[sl], w[h:][sl], w[2 * h:][sl]], axis=0))
    return np.stack(parts)


def unshard_qkv_rows(ws: np.ndarray) -> np.ndarray:
    t, rows = ws.shape[0], ws.shape[1]
    hs = rows // 3
    q = np.concatenate([ws[i, :hs] for i in range(t)])
    k = np.concatenate([ws[i, hs:2 * hs] for i in range(t)])
    v = np.concatenate([ws[i, 2 * hs:] for i in range(t)])
    return np.concatenate([q, k, v])


def shard_rows(w: np.ndarray, t: int) -> np.ndarray:
    """Column-split (output) dimension: [n, ...] -> [t, n/t, ...]."""
    return np.ascontiguousarray(w.reshape((t, w.shape[0] // t) + w.shape[1:]))


def shard_cols(w: np.ndarray, t: int) -> np.ndarray:
    """Row-split (input) dimension: [n_out, n_in] -> [t, n_out, n_in/t]."""
    n_out, n_in = w.shape
    return np.ascontiguousarray(w.reshape(n_out, t, n_in // t).transpose(1, 0, 2))


def unshard_cols(ws: np.ndarray) -> np.ndarray:
    t, n_out, k = ws.shape
    return np.ascontiguousarray(ws.transpose(1, 0, 2).reshape(n_out, t * k))


def shard_params(u: dict, t: int) -> dict:
    """Unsharded [out, in] parameters -> the shard-major layout."""
    return {
        "ln1_g": u["ln1_g"], "ln1_b": u["ln1_b"],
        "w_qkv": shard_qkv_rows(u["w_qkv"], t), "b_qkv": shard_qkv_rows(u["b_qkv"], t),
        "w_o": shard_cols(u["w_o"], t), "b_o": u["b_o"],
        "ln2_g": u["ln2_g"], "ln2_b": u["ln2_b"],
        "w_1": shard_rows(u["w_1"], t), "b_1": shard_rows(u["b_1"], t),
        "w_2": shard_cols(u["w_2"], t), "b_2": u["b_2"],
    }


def unshard_params(p: dict) -> dict:
    return {
        "ln1_g": p["ln1_g"], "ln1_b": p["ln1_b"],
        "w_qkv": unshard_qkv_rows(p["w_qkv"]), "b_qkv": unshard_qkv_rows(p["b_qkv"]),
        "w_o": unshard_cols(p["w_o"]), "b_o": p["b_o"],
        "ln2_g": p["ln2_g"], "ln2_b": p["ln2_b"],
        "w_1": p["w_1"].reshape((-1,) + p["w_1"].shape[2:]),
        "b_1": p["b_1"].reshape(-1),
        "w_2": unshard_cols(p["w_2"]), "b_2": p["b_2"],
    }


# --------------------------------------------------------------------------
# Draws
# --------------------------------------------------------------------------
def _normal(rng, shape, std, dtype, chunk_rows=4096):
    """Normal draw rounded to the 16-bit type, in row chunks to bound memory."""
    shape = tuple(shape)
    out = np.empty(shape, dtype=np.uint16)
    flat = out.reshape(shape[0], -1)
    for r0 in range(0, shape[0], chunk_rows):
        r1 = min(shape[0], r0 + chunk_rows)
        flat[r0:r1] = to_bits(rng.standard_normal((r1 - r0, flat.shape[1])) * std, dtype)
    return out


def make_inputs(cfg: LayerConfig, seed: int = 0, variant: str = "plain",
                with_r: bool = False) -> dict:
    """Seeded inputs as uint16 bit patterns.

    Returns {"x": [T,h], "params": shard-major dict, "r": [T,h] or None}.
    variant "plain": biases 0, gamma 1, beta 0.  variant "biased": every bias,
    gamma-1 and beta drawn N(0, 0.02) so that each path carries signal.
    """
    rng = np.random.default_rng(seed)
    h, f, t, T = cfg.hidden, cfg.ffn, cfg.tp, cfg.tokens
    dt = cfg.dtype
    x = _normal(rng, (T, h), 1.0, dt)
    u = {
        "w_qkv": _normal(rng, (3 * h, h), cfg.w_std, dt),
        "w_o": _normal(rng, (h, h), cfg.w_std, dt),
        "w_1": _normal(rng, (f, h), cfg.w_std, dt),
        "w_2": _normal(rng, (h, f), cfg.w_std, dt),
    }
    one = to_bits(np.ones(h), dt)
    zero_h = to_bits(np.zeros(h), dt)
    if variant == "plain":
        u.update(b_qkv=to_bits(np.zeros(3 * h), dt), b_o=zero_h.copy(),
                 b_1=to_bits(np.zeros(f), dt), b_2=zero_h.copy(),
                 ln1_g=one.copy(), ln1_b=zero_h.copy(),
                 ln2_g=one.copy(), ln2_b=zero_h.copy())
    elif variant == "biased":
        u["b_qkv"] = to_bits(rng.standard_normal(3 * h) * 0.02, dt)
        u["b_o"] = to_bits(rng.standard_normal(h) * 0.02, dt)
        u["b_1"] = to_bits(rng.standard_normal(f) * 0.02, dt)
        u["b_2"] = to_bits(rng.standard_normal(h) * 0.02, dt)
        u["ln1_g"] = to_bits(1.0 + rng.standard_normal(h) * 0.02, dt)
        u["ln1_b"] = to_bits(rng.standard_normal(h) * 0.02, dt)
        u["ln2_g"] = to_bits(1.0 + rng.standard_normal(h) * 0.02, dt)
        u["ln2_b"] = to_bits(rng.standard_normal(h) * 0.02, dt)
    else:
        raise ValueError(variant)
    r = _normal(rng, (T, h), 1.0, dt) if with_r else None
    return {"x": x, "params": shard_params(u, t), "r": r}


def loss_grad_bits(cfg: LayerConfig, scale: float, r_bits=None) -> np.ndarray:
    """dOut for loss = mean(Out) (or mean(Out * R)), multiplied by the loss
    scale, rounded to the 16-bit type.  This is the harness's loss, not part
    of the layer."""
    T, h = cfg.tokens, cfg.hidden
    if r_bits is None:
        g = np.full((T, h), scale / (T * h))
    else:
        g = from_bits(r_bits, cfg.dtype) * (scale / (T * h))
    return to_bits(g, cfg.dtype)


def random_fp32(n: int, seed: int, std: float = 1.0) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.standard_normal(n) * std).astype(np.float32)
