"""Mixed-precision optimizer side of the step: overflow check, Adam on FP32
master weights, dynamic loss-scale update.  Test infrastructure only.

"Megatron-LM overview" §3.1: matrices are multiplied in FP16, an FP32 master
copy of the weights receives the update, and the loss is scaled
dynamically.  §4.2 names Adam with lr 6e-5.  §5.1 advises adjusting the
initial scale when loss scaling misbehaves, and names gradient clipping
that is too strong as a cause of non-convergence.  "Training GPT-2 with
Megatron-LM" §4.3 accumulates gradients over micro-batches
(--gradient-accumulation-steps) and its troubleshooting list adds
--clip-grad 1.0 against NaN losses.

Readings where the pages are silent:
  * overflow: any inf or NaN in the (scaled) fp32 gradients;
  * skipped step: master, m, v and the 16-bit copy untouched, step count
    not advanced;
  * Adam: bias-corrected, eps outside the square root, decoupled weight
    decay (0 by default);
  * scaler: back off on the first overflow (no hysteresis), floor
    min_scale, multiply by growth_factor after growth_interval clean steps;
  * clipping: by the global L2 norm of the unscaled gradient over the whole
    parameter arena, coefficient max_norm / (norm + 1e-6) applied when it is
    below 1 (the usual global-norm clip; the pages give only the threshold);
  * accumulation: the gradients of the micro-batches are summed in fp32
    (the gradient of the summed loss); averaging, if wanted, belongs to the
    loss gradient that the caller feeds to the backward pass.
"""
from __future__ import annotations

import numpy as np


def found_inf(*grads: np.ndarray) -> int:
    """1 if any element of any fp32 gradient array is inf or NaN (all
    exponent bits set), else 0."""
    for g in grads:
        bits = np.ascontiguousarray(g, dtype=np.float32).view(np.uint32)
        if np.any((bits & 0x7F800000) == 0x7F800000):
            return 1
    return 0


def cast_to_16(p: np.ndarray, dtype: str) -> np.ndarray:
    """Round-to-nearest-even of float64 values into fp16 or bf16, returned as
    uint16 bit patterns.

    bf16 keeps the top 16 bits of an fp32 pattern, so the value is first
    brought to fp32 exactly when it is representable; the rounding of the
    remaining bits is done here bit by bit from the float64 value to avoid a
    double rounding."""
    p = np.asarray(p, dtype=np.float64)
    if dtype == "fp16":
        return p.astype(np.float16).view(np.uint16)
    if dtype == "bf16":
        # bf16 grid: 8 significant bits.  Scale each value to an integer
        # significand and round half to even in float64 arithmetic.
        out = np.zeros(p.shape, dtype=np.uint16)
        flat_p = p.reshape(-1)
        flat_o = out.reshape(-1)
        finite = np.isfinite(flat_p) & (flat_p != 0)
        v = flat_p[finite]
        e = np.floor(np.log2(np.abs(v)))
        # guard against log2 rounding at exact powers of two
        e = np.where(np.abs(v) >= 2.0 ** (e + 1), e + 1, e)
        e = np.where(np.abs(v) < 2.0 ** e, e - 1, e)
        e = np.maximum(e, -126.0)               # bf16 subnormals share fp32's range
        ulp = 2.0 ** (e - 7)
        q = np.round(v / ulp) * ulp             # np.round is half-to-even
        flat_o[finite] = (np.asarray(q, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
        zero = flat_p == 0
        flat_o[zero] = np.where(np.signbit(flat_p[zero]), 0x8000, 0).astype(np.uint16)
        flat_o[np.isnan(flat_p)] = 0x7FC0
        flat_o[np.isposinf(flat_p)] = 0x7F80
        flat_o[np.isneginf(flat_p)] = 0xFF80
        return out
    raise ValueError(dtype)


def round_to_16(x: np.ndarray, dtype: str) -> np.ndarray:
    """float64 value of the fp16/bf16 number nearest to x (ties to even):
    the value a 16-bit activation tensor holds once stored."""
    bits = cast_to_16(x, dtype)
    if dtype == "fp16":
        return bits.view(np.float16).astype(np.float64)
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def grad_norm(grad: np.ndarray, scale: float) -> float:
    """Global L2 norm of the unscaled gradient, sqrt(sum_i (grad_i / S)^2),
    in float64 from the fp32 (scaled) gradient arena."""
    g = np.asarray(grad, dtype=np.float64).reshape(-1) / scale
    return float(np.sqrt(np.dot(g, g)))


def clip_coefficient(norm: float, max_norm: float) -> float:
    """Factor applied to the unscaled gradient by global-norm clipping:
    max_norm / (norm + 1e-6) when that is below 1, else exactly 1."""
    c = max_norm / (norm + 1e-6)
    return c if c < 1.0 else 1.0


def accumulate(acc: np.ndarray, grad: np.ndarray) -> np.ndarray:
    """acc + grad rounded to fp32 (one fp32 addition per element).  The
    float64 sum of two fp32 numbers rounds to the same fp32 value as the
    fp32 addition, so this is the exact fp32 result."""
    return (np.asarray(acc, dtype=np.float32).astype(np.float64) +
            np.asarray(grad, dtype=np.float32).astype(np.float64)).astype(np.float32)


def adam_step(master: np.ndarray, m: np.ndarray, v: np.ndarray, grad: np.ndarray,
              scale: float, step: int, lr: float, beta1: float, beta2: float,
              eps: float, weight_decay: float, dtype: str, inf_flag: int,
              clip_coef: float = 1.0):
    """One Adam update on FP32 masters, computed in float64 from the fp32
    inputs.  `step` is the number of steps taken so far (t = step + 1).
    The unscaled gradient grad / scale is multiplied by clip_coef (from
    clip_coefficient; 1 without clipping) before it enters the moments.

    Returns (master, m, v, w16_bits) as float64/float64/float64/uint16; on
    overflow (inf_flag == 1) returns the inputs unchanged and w16 = None."""
    if inf_flag:
        return master, m, v, None
    p = np.asarray(master, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    g = np.asarray(grad, dtype=np.float64) / scale * clip_coef
    t = step + 1
    m_new = beta1 * m + (1.0 - beta1) * g
    v_new = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m_new / (1.0 - beta1 ** t)
    v_hat = v_new / (1.0 - beta2 ** t)
    p_new = p - lr * (m_hat / (np.sqrt(v_hat) + eps) + weight_decay * p)
    return p_new, m_new, v_new, cast_to_16(p_new, dtype)


def loss_scale_update(state: dict, inf_flag: int, growth_interval: int,
                      growth_factor: float, backoff_factor: float,
                      min_scale: float) -> dict:
    """Dynamic loss-scale rule.  state = {scale, growth_tracker, step}."""
    s = dict(state)
    if inf_flag:
        s["scale"] = max(s["scale"] * backoff_factor, min_scale)
        s["growth_tracker"] = 0
    else:
        s["growth_tracker"] += 1
        if s["growth_tracker"] == growth_interval:
            s["scale"] = s["scale"] * growth_factor
            s["growth_tracker"] = 0
        s["step"] += 1
    return s
