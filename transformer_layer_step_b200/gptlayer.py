"""ctypes binding of libgptlayer.so (declared in include/gptlayer.h,
include/gptlayer_parts.h and include/gptlayer_profile.h).

Argument marshalling only: every computation happens in the library's CUDA
kernels.  Pointers are passed as integers (or objects with .data_ptr(), such
as torch tensors); streams as the integer handle of a cudaStream_t.  A
non-zero return code raises GptlError.  If the library has not been built the
first call raises at once: there is no fallback path.
"""
from __future__ import annotations

import ctypes as C
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libgptlayer.so")
INCLUDE = os.path.join(os.path.dirname(PKG), "include")

FP16, BF16 = 0, 1
ACT_NONE, ACT_GELU, ACT_DGELU = 0, 1, 2
E_NULL, E_SHAPE, E_ALIGN, E_DTYPE, E_ARCH, E_CUDA, E_DEVICE, E_ARG = -1, -2, -3, -4, -5, -6, -7, -8
E_TOO_LARGE = -9
DTYPES = {"fp16": FP16, "bf16": BF16}
PARAM_NAMES = ("ln1_g", "ln1_b", "w_qkv", "b_qkv", "w_o", "b_o",
               "ln2_g", "ln2_b", "w_1", "b_1", "w_2", "b_2")
# optional transposed copies of the four weight matrices (gptl_weights)
WT_NAMES = ("w_qkv_t", "w_o_t", "w_1_t", "w_2_t")


class GptlError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} ({code})")


class Shape(C.Structure):
    _fields_ = [("batch", C.c_int), ("seq", C.c_int), ("hidden", C.c_int), ("heads", C.c_int),
                ("ffn", C.c_int), ("tp", C.c_int), ("dtype", C.c_int), ("ln_eps", C.c_float),
                ("recompute_gelu", C.c_int)]


class Weights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in PARAM_NAMES + WT_NAMES]


class Grads(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in PARAM_NAMES]


class ScalerState(C.Structure):
    _fields_ = [("scale", C.c_float), ("growth_tracker", C.c_int), ("found_inf", C.c_int),
                ("step", C.c_int), ("error", C.c_int)]


class Operand(C.Structure):
    _fields_ = [("ptr", C.c_void_p), ("x_ext", C.c_longlong), ("rows_ext", C.c_longlong),
                ("g_ext", C.c_longlong), ("row_pitch", C.c_longlong), ("g_pitch", C.c_longlong),
                ("mn_major", C.c_int), ("x_mod", C.c_int), ("x_mul", C.c_int), ("x_off", C.c_int),
                ("g_div", C.c_int), ("k_shard", C.c_int)]


class GemmDesc(C.Structure):
    _fields_ = [("M", C.c_int), ("N", C.c_int), ("K", C.c_int), ("groups", C.c_int),
                ("k_shards", C.c_int), ("causal", C.c_int), ("a", Operand), ("b", Operand),
                ("out", C.c_void_p), ("out_f32", C.c_int), ("ldo", C.c_longlong),
                ("o_mod", C.c_int), ("o_str_mod", C.c_longlong), ("o_str_div", C.c_longlong),
                ("bias", C.c_void_p), ("bias_g_stride", C.c_longlong), ("resid", C.c_void_p),
                ("ld_resid", C.c_longlong), ("aux", C.c_void_p), ("out2", C.c_void_p),
                ("act", C.c_int), ("resid_f32", C.c_int), ("ws", C.c_void_p),
                ("ws_bytes", C.c_longlong), ("colsum", C.c_void_p)]


class LaunchRecord(C.Structure):
    _fields_ = [("kind", C.c_int), ("tag", C.c_int), ("ms", C.c_float)]


KIND_NAMES = ("gemm", "ln_fwd", "ln_bwd", "reserved3", "reserved4", "colsum", "reduce",
              "overflow", "adam", "scale", "splitk", "attn_fwd", "rowdot", "transpose", "attn_bwd",
              "clip", "accumulate")

_lib = None

_SIGS = {
    "gptl_strerror": (C.c_char_p, [C.c_int]),
    "gptl_read_device_error": (C.c_int, [C.POINTER(C.c_int), C.c_int]),
    "gpt_layer_workspace_bytes": (C.c_int, [C.POINTER(Shape), C.POINTER(C.c_size_t),
                                            C.POINTER(C.c_size_t)]),
    "gpt_layer_param_layout": (C.c_int, [C.POINTER(Shape), C.POINTER(C.c_size_t),
                                         C.POINTER(C.c_size_t)]),
    "gpt_layer_fwd": (C.c_int, [C.POINTER(Shape), C.POINTER(Weights), C.c_void_p, C.c_void_p,
                                C.c_void_p, C.c_void_p, C.c_void_p]),
    "gpt_layer_bwd": (C.c_int, [C.POINTER(Shape), C.POINTER(Weights), C.c_void_p, C.c_void_p,
                                C.c_void_p, C.c_void_p, C.POINTER(Grads), C.c_void_p, C.c_void_p]),
    "gpt_layer_bwd_checked": (C.c_int, [C.POINTER(Shape), C.POINTER(Weights), C.c_void_p,
                                        C.c_void_p, C.c_void_p, C.c_void_p, C.POINTER(Grads),
                                        C.c_void_p, C.c_void_p, C.c_void_p]),
    "adam_step_fp32_master_prechecked": (C.c_int, [C.c_size_t, C.c_void_p, C.c_void_p,
                                                   C.c_void_p, C.c_void_p, C.c_void_p, C.c_int,
                                                   C.c_float, C.c_float, C.c_float, C.c_float,
                                                   C.c_float, C.c_void_p, C.c_void_p]),
    "gpt_layer_adam_step": (C.c_int, [C.POINTER(Shape), C.c_int] + [C.c_void_p] * 6 +
                            [C.c_float] * 5 + [C.c_int, C.c_void_p, C.c_void_p]),
    "gpt_layer_transpose_weights": (C.c_int, [C.POINTER(Shape), C.c_int, C.c_void_p, C.c_void_p,
                                              C.c_void_p]),
    "gpt_stack_workspace_bytes": (C.c_int, [C.POINTER(Shape), C.c_int, C.POINTER(C.c_size_t),
                                            C.POINTER(C.c_size_t)]),
    "gpt_stack_fwd": (C.c_int, [C.POINTER(Shape), C.c_int, C.POINTER(Weights), C.c_void_p,
                                C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "gpt_stack_bwd": (C.c_int, [C.POINTER(Shape), C.c_int, C.POINTER(Weights), C.c_void_p,
                                C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.POINTER(Grads),
                                C.c_void_p, C.c_void_p]),
    "adam_step_fp32_master": (C.c_int, [C.c_size_t, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                        C.c_void_p, C.c_int, C.c_float, C.c_float, C.c_float,
                                        C.c_float, C.c_float, C.c_void_p, C.c_void_p]),
    "loss_scale_update": (C.c_int, [C.c_void_p, C.c_int, C.c_float, C.c_float, C.c_float,
                                    C.c_void_p]),
    "gptl_check_overflow": (C.c_int, [C.c_size_t, C.c_void_p, C.c_void_p, C.c_void_p]),
    "adam_step_fp32_master_clip": (C.c_int, [C.c_size_t, C.c_void_p, C.c_void_p, C.c_void_p,
                                             C.c_void_p, C.c_void_p, C.c_int, C.c_float,
                                             C.c_float, C.c_float, C.c_float, C.c_float,
                                             C.c_float, C.c_void_p, C.c_void_p, C.c_void_p]),
    "gptl_grad_accumulate": (C.c_int, [C.c_size_t, C.c_void_p, C.c_void_p, C.c_void_p]),
    "gptl_gemm": (C.c_int, [C.POINTER(GemmDesc), C.c_int, C.c_void_p]),
    "gptl_gemm_plan": (C.c_int, [C.POINTER(GemmDesc), C.c_int, C.POINTER(C.c_int),
                                 C.POINTER(C.c_int), C.POINTER(C.c_int)]),
    "gptl_layernorm_fwd": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p]),
    "gptl_layernorm_bwd_scratch_bytes": (C.c_size_t, [C.c_int, C.c_int]),
    "gptl_layernorm_bwd": (C.c_int, [C.c_int, C.c_int, C.c_int] + [C.c_void_p] * 11 + [C.c_void_p]),
    "gptl_colsum_scratch_bytes": (C.c_size_t, [C.c_int, C.c_int]),
    "gptl_colsum": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_longlong, C.c_longlong, C.c_int,
                              C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "gptl_attention_fwd": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_int, C.c_int, C.c_int,
                                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "gptl_attention_bwd": (C.c_int, [C.c_int] * 6 + [C.c_void_p] * 9),
    "gptl_colsum_noalloc": (C.c_int, [C.c_int, C.c_int, C.c_int, C.c_longlong, C.c_longlong,
                                      C.c_int, C.c_void_p, C.c_void_p, C.c_void_p]),
    "gptl_launch_count": (C.c_ulonglong, []),
    "gptl_profile_begin": (C.c_int, [C.c_int]),
    "gptl_profile_end": (C.c_int, [C.POINTER(LaunchRecord), C.c_int, C.POINTER(C.c_int),
                                   C.POINTER(C.c_longlong)]),
    "gptl_tag_name": (C.c_char_p, [C.c_int]),
}


def lib():
    """The loaded library (loaded on first use; raises if it is not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run `python -m transformer_layer_step_b200.build`"
                               " (there is no fallback implementation)")
        handle = C.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def header_functions() -> list:
    """Names of every function declared in include/*.h."""
    names = []
    for fname in sorted(os.listdir(INCLUDE)):
        if not fname.endswith(".h"):
            continue
        text = open(os.path.join(INCLUDE, fname)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z_0-9]*\s*\*?\s*([a-z_][a-z_0-9]*)\s*\(",
                            text, flags=re.M)
    return sorted(set(names))


def strerror(code: int) -> str:
    return lib().gptl_strerror(code).decode()


def _ptr(x) -> int | None:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _check(rc: int, where: str):
    if rc != 0:
        raise GptlError(rc, where)


def make_shape(batch, seq, hidden, heads, ffn, tp, dtype, ln_eps=1e-5, recompute_gelu=0) -> Shape:
    return Shape(batch, seq, hidden, heads, ffn, tp, DTYPES.get(dtype, dtype), ln_eps,
                 int(recompute_gelu))


def workspace_bytes(shape: Shape):
    a, b = C.c_size_t(), C.c_size_t()
    _check(lib().gpt_layer_workspace_bytes(C.byref(shape), C.byref(a), C.byref(b)),
           "gpt_layer_workspace_bytes")
    return a.value, b.value


def param_layout(shape: Shape):
    offs = (C.c_size_t * 12)()
    n = C.c_size_t()
    _check(lib().gpt_layer_param_layout(C.byref(shape), offs, C.byref(n)), "gpt_layer_param_layout")
    return [int(o) for o in offs], n.value


def make_weights(ptrs: dict) -> Weights:
    """ptrs: the 12 parameter pointers, and optionally the 4 WT_NAMES copies."""
    return Weights(*[_ptr(ptrs[n]) for n in PARAM_NAMES], *[_ptr(ptrs.get(n)) for n in WT_NAMES])


def make_grads(ptrs: dict) -> Grads:
    return Grads(*[_ptr(ptrs[n]) for n in PARAM_NAMES])


def layer_fwd(shape, weights: Weights, x, y, saved, scratch=None, stream=0):
    _check(lib().gpt_layer_fwd(C.byref(shape), C.byref(weights), _ptr(x), _ptr(y), _ptr(saved),
                               _ptr(scratch), stream), "gpt_layer_fwd")


def layer_bwd(shape, weights: Weights, x, saved, dy, dx, grads: Grads, scratch, stream=0):
    _check(lib().gpt_layer_bwd(C.byref(shape), C.byref(weights), _ptr(x), _ptr(saved), _ptr(dy),
                               _ptr(dx), C.byref(grads), _ptr(scratch), stream), "gpt_layer_bwd")


def layer_bwd_checked(shape, weights: Weights, x, saved, dy, dx, grads: Grads, scratch, state,
                      stream=0):
    """gpt_layer_bwd that also sets state.found_inf from the gradients it writes."""
    _check(lib().gpt_layer_bwd_checked(C.byref(shape), C.byref(weights), _ptr(x), _ptr(saved),
                                       _ptr(dy), _ptr(dx), C.byref(grads), _ptr(scratch),
                                       _ptr(state), stream), "gpt_layer_bwd_checked")


def stack_workspace_bytes(shape: Shape, n_layers: int):
    a, b = C.c_size_t(), C.c_size_t()
    _check(lib().gpt_stack_workspace_bytes(C.byref(shape), n_layers, C.byref(a), C.byref(b)),
           "gpt_stack_workspace_bytes")
    return a.value, b.value


def stack_fwd(shape, weights, x, acts, saved, scratch=None, stream=0):
    """weights: a sequence of Weights, one per layer; scratch: needed when the
    shape has recompute_gelu."""
    arr = (Weights * len(weights))(*weights)
    _check(lib().gpt_stack_fwd(C.byref(shape), len(weights), arr, _ptr(x), _ptr(acts),
                               _ptr(saved), _ptr(scratch), stream), "gpt_stack_fwd")


def stack_bwd(shape, weights, x, acts, saved, dy, dx, grads, scratch, stream=0):
    """weights, grads: sequences of Weights / Grads, one per layer."""
    if len(grads) != len(weights):
        raise ValueError("one Grads per layer")
    wa = (Weights * len(weights))(*weights)
    ga = (Grads * len(grads))(*grads)
    _check(lib().gpt_stack_bwd(C.byref(shape), len(weights), wa, _ptr(x), _ptr(acts), _ptr(saved),
                               _ptr(dy), _ptr(dx), ga, _ptr(scratch), stream), "gpt_stack_bwd")


def adam_step(n_params, master, m, v, grad, w16, dtype, lr, beta1, beta2, eps, weight_decay,
              state, stream=0):
    _check(lib().adam_step_fp32_master(n_params, _ptr(master), _ptr(m), _ptr(v), _ptr(grad),
                                       _ptr(w16), DTYPES.get(dtype, dtype), lr, beta1, beta2, eps,
                                       weight_decay, _ptr(state), stream), "adam_step_fp32_master")


def layer_adam_step(shape, n_layers, master, m, v, grad, w16, w16t, lr, beta1, beta2, eps,
                    weight_decay, prechecked, state, stream=0):
    """gpt_layer_adam_step: the optimizer step that also writes the transposed
    weight matrices of n_layers layer arenas into w16t."""
    _check(lib().gpt_layer_adam_step(C.byref(shape), n_layers, _ptr(master), _ptr(m), _ptr(v),
                                     _ptr(grad), _ptr(w16), _ptr(w16t), lr, beta1, beta2, eps,
                                     weight_decay, int(prechecked), _ptr(state), stream),
           "gpt_layer_adam_step")


def transpose_weights(shape, n_layers, w16, w16t, stream=0):
    _check(lib().gpt_layer_transpose_weights(C.byref(shape), n_layers, _ptr(w16), _ptr(w16t), stream),
           "gpt_layer_transpose_weights")


def adam_step_prechecked(n_params, master, m, v, grad, w16, dtype, lr, beta1, beta2, eps,
                         weight_decay, state, stream=0):
    """adam_step_fp32_master taking state.found_inf as gpt_layer_bwd_checked left it."""
    _check(lib().adam_step_fp32_master_prechecked(n_params, _ptr(master), _ptr(m), _ptr(v),
                                                  _ptr(grad), _ptr(w16), DTYPES.get(dtype, dtype),
                                                  lr, beta1, beta2, eps, weight_decay, _ptr(state),
                                                  stream), "adam_step_fp32_master_prechecked")


# bytes of the clip workspace (GPTL_CLIP_WORKSPACE_BYTES in gptlayer.h); the
# norm of the unscaled gradient is the float at byte 0, the clip coefficient
# the float at byte 4
CLIP_WORKSPACE_BYTES = 16384


def adam_step_clip(n_params, master, m, v, grad, w16, dtype, lr, beta1, beta2, eps, weight_decay,
                   max_norm, clip_ws, state, stream=0):
    _check(lib().adam_step_fp32_master_clip(n_params, _ptr(master), _ptr(m), _ptr(v), _ptr(grad),
                                            _ptr(w16), DTYPES.get(dtype, dtype), lr, beta1, beta2,
                                            eps, weight_decay, max_norm, _ptr(clip_ws),
                                            _ptr(state), stream),
           "adam_step_fp32_master_clip")


def grad_accumulate(n, acc, grad, stream=0):
    _check(lib().gptl_grad_accumulate(n, _ptr(acc), _ptr(grad), stream), "gptl_grad_accumulate")


def scale_update(state, growth_interval, growth_factor, backoff_factor, min_scale, stream=0):
    _check(lib().loss_scale_update(_ptr(state), growth_interval, growth_factor, backoff_factor,
                                   min_scale, stream), "loss_scale_update")


def check_overflow(n, grad, state, stream=0):
    _check(lib().gptl_check_overflow(n, _ptr(grad), _ptr(state), stream), "gptl_check_overflow")


def operand(t, x_ext, rows_ext, g_ext, row_pitch, g_pitch=0, mn_major=0, x_mod=1, x_mul=0,
            x_off=0, g_div=None, k_shard=0) -> Operand:
    if g_div is None:
        g_div = 1 if g_ext > 1 else (1 << 30)
    return Operand(_ptr(t), x_ext, rows_ext, g_ext, row_pitch, g_pitch, mn_major, x_mod, x_mul,
                   x_off, g_div, k_shard)


def gemm(desc: GemmDesc, dtype, stream=0):
    _check(lib().gptl_gemm(C.byref(desc), DTYPES.get(dtype, dtype), stream), "gptl_gemm")


GEMM_ALTERNATE, GEMM_K_HALVES, GEMM_M256 = 0, 1, 2


def gemm_plan(desc: GemmDesc, dtype) -> tuple:
    """(bn, split, mode) that gptl_gemm would use for desc on this device."""
    bn, split, mode = C.c_int(), C.c_int(), C.c_int()
    _check(lib().gptl_gemm_plan(C.byref(desc), DTYPES.get(dtype, dtype), C.byref(bn),
                                C.byref(split), C.byref(mode)), "gptl_gemm_plan")
    return bn.value, split.value, mode.value


def layernorm_fwd(rows, h, dtype, x, g, b, eps, y, mu, rstd, stream=0):
    _check(lib().gptl_layernorm_fwd(rows, h, DTYPES.get(dtype, dtype), _ptr(x), _ptr(g), _ptr(b),
                                    eps, _ptr(y), _ptr(mu), _ptr(rstd), stream), "gptl_layernorm_fwd")


def layernorm_bwd_scratch_bytes(rows, h) -> int:
    return lib().gptl_layernorm_bwd_scratch_bytes(rows, h)


def layernorm_bwd(rows, h, dtype, gy, x, mu, rstd, g, resid, dx, dg, db, dx_sum, scratch, stream=0):
    _check(lib().gptl_layernorm_bwd(rows, h, DTYPES.get(dtype, dtype), _ptr(gy), _ptr(x), _ptr(mu),
                                    _ptr(rstd), _ptr(g), _ptr(resid), _ptr(dx), _ptr(dg), _ptr(db),
                                    _ptr(dx_sum), _ptr(scratch), stream), "gptl_layernorm_bwd")


def colsum_scratch_bytes(n, groups) -> int:
    return lib().gptl_colsum_scratch_bytes(n, groups)


def colsum(rows, n, groups, ld, gstride, dtype, a, out, scratch, stream=0):
    _check(lib().gptl_colsum(rows, n, groups, ld, gstride, DTYPES.get(dtype, dtype), _ptr(a),
                             _ptr(out), _ptr(scratch), stream), "gptl_colsum")


def attention_fwd(batch, seq, hidden, heads, tp, dtype, qkv, o, lse, stream=0):
    _check(lib().gptl_attention_fwd(batch, seq, hidden, heads, tp, DTYPES.get(dtype, dtype), _ptr(qkv),
                                    _ptr(o), _ptr(lse), stream), "gptl_attention_fwd")


def attention_bwd(batch, seq, hidden, heads, tp, dtype, qkv, o, dout, lse, dvec, dqkv,
                  dbias_part=None, dbias=None, stream=0):
    _check(lib().gptl_attention_bwd(batch, seq, hidden, heads, tp, DTYPES.get(dtype, dtype), _ptr(qkv),
                                    _ptr(o), _ptr(dout), _ptr(lse), _ptr(dvec), _ptr(dqkv),
                                    _ptr(dbias_part), _ptr(dbias), stream),
           "gptl_attention_bwd")


def colsum_noalloc(rows, n, groups, ld, gstride, dtype, a, out, stream=0):
    """gptl_colsum without caller scratch (fixed library array; see the header)."""
    _check(lib().gptl_colsum_noalloc(rows, n, groups, ld, gstride, DTYPES.get(dtype, dtype),
                                     _ptr(a), _ptr(out), stream), "gptl_colsum_noalloc")


def read_device_error(clear: bool = True) -> int:
    w = C.c_int()
    _check(lib().gptl_read_device_error(C.byref(w), 1 if clear else 0), "gptl_read_device_error")
    return w.value


def launch_count() -> int:
    """Kernels launched through the library by this process so far."""
    return int(lib().gptl_launch_count())


def profile_begin(capacity: int):
    _check(lib().gptl_profile_begin(capacity), "gptl_profile_begin")


def profile_end(capacity: int):
    """Closes the profiling window; returns ([(kind_name, tag_name, ms)], dropped)."""
    recs = (LaunchRecord * capacity)()
    n, dropped = C.c_int(), C.c_longlong()
    _check(lib().gptl_profile_end(recs, capacity, C.byref(n), C.byref(dropped)),
           "gptl_profile_end")
    out = [(KIND_NAMES[r.kind], lib().gptl_tag_name(r.tag).decode(), float(r.ms))
           for r in recs[:n.value]]
    return out, int(dropped.value)
