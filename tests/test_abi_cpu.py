"""The C-ABI library loads without a GPU, exports every function that
include/*.h declares, and rejects bad arguments before touching the device."""
import ctypes

import pytest

from transformer_layer_step_b200 import gptlayer as G
from transformer_layer_step_b200 import synth


def test_exports_every_declared_function():
    lib = G.lib()
    declared = G.header_functions()
    assert "gpt_layer_fwd" in declared and "adam_step_fp32_master" in declared
    for name in declared:
        assert hasattr(lib, name), name


def test_strerror_codes():
    for code in (0, G.E_NULL, G.E_SHAPE, G.E_ALIGN, G.E_DTYPE, G.E_ARCH, G.E_CUDA, G.E_DEVICE, G.E_ARG,
                 G.E_TOO_LARGE):
        assert G.strerror(code) and G.strerror(code) != "unknown error"


@pytest.mark.parametrize("name", list(synth.CONFIGS))
def test_workspace_and_layout(name):
    c = synth.CONFIGS[name]
    sh = G.make_shape(c.batch, c.seq, c.hidden, c.heads, c.ffn, c.tp, c.dtype)
    saved, scratch = G.workspace_bytes(sh)
    T, h, f = c.tokens, c.hidden, c.ffn
    # the residual stream H (saved) and its gradient dH (scratch) are fp32;
    # the attention keeps a row log-sum-exp (saved) and recomputes P in the
    # backward (scratch holds P and dS)
    rows = c.batch * c.heads * c.seq
    assert saved >= 2 * (T * h * 7 + 2 * T * f) + 4 * rows
    assert scratch >= 2 * T * f + 20 * T * h + 4 * rows
    offs, n = G.param_layout(sh)
    sizes = [h, h, 3 * h * h, 3 * h, h * h, h, h, h, f * h, f, h * f, h]
    assert n % 64 == 0 and all(o % 64 == 0 for o in offs)
    for i in range(11):
        assert offs[i] + sizes[i] <= offs[i + 1]
    assert offs[11] + sizes[11] <= n
    assert n - sum(sizes) < 64 * 12
    assert sum(sizes) == 12 * h * h + 13 * h


@pytest.mark.parametrize("bad", [
    dict(heads=5),                 # heads does not divide hidden
    dict(tp=3),                    # tp does not divide heads
    dict(hidden=96, heads=2),      # hidden not a multiple of 64
    dict(seq=72),                  # seq not a multiple of 16
    dict(heads=16),                # head_dim 8, not a multiple of 16
    dict(hidden=2048, heads=8, ffn=8192),   # head_dim 256, above the attention kernel's 128
    dict(batch=0),
    dict(seq=4096),                # beyond the supported sequence length
])
def test_shape_validation(bad):
    args = dict(batch=2, seq=64, hidden=128, heads=4, ffn=512, tp=2, dtype="fp16")
    args.update(bad)
    sh = G.make_shape(**args)
    with pytest.raises(G.GptlError) as e:
        G.workspace_bytes(sh)
    assert e.value.code == G.E_SHAPE


def test_dtype_and_null_rejected_without_launch():
    sh = G.make_shape(2, 64, 128, 4, 512, 2, 7)
    with pytest.raises(G.GptlError) as e:
        G.workspace_bytes(sh)
    assert e.value.code == G.E_DTYPE
    sh = G.make_shape(2, 64, 128, 4, 512, 2, "fp16")
    w = G.Weights()
    rc = G.lib().gpt_layer_fwd(ctypes.byref(sh), ctypes.byref(w), 16, 16, 16, None, None)
    assert rc == G.E_NULL
    rc = G.lib().adam_step_fp32_master(64, 16, 16, 16, 16, 16, 0, -1.0, 0.9, 0.95, 1e-8, 0.0, 16, None)
    assert rc == G.E_ARG
    rc = G.lib().adam_step_fp32_master(64, 17, 16, 16, 16, 16, 0, 1e-3, 0.9, 0.95, 1e-8, 0.0, 16, None)
    assert rc == G.E_ALIGN
    rc = G.lib().loss_scale_update(16, 0, 2.0, 0.5, 1.0, None)
    assert rc == G.E_ARG
    # recompute_gelu: the forward writes A into scratch, so it needs scratch
    shr = G.make_shape(2, 64, 128, 4, 512, 2, "fp16", recompute_gelu=1)
    rc = G.lib().gpt_layer_fwd(ctypes.byref(shr), ctypes.byref(w), 16, 16, 16, None, None)
    assert rc == G.E_NULL
    # the attention backward's bias gradient needs both its partials and its output
    rc = G.lib().gptl_attention_bwd(1, 64, 128, 4, 1, 0, 16, 16, 16, 16, 16, 16, None, 16, None)
    assert rc == G.E_NULL
    rc = G.lib().gptl_attention_bwd(1, 64, 128, 4, 1, 0, 16, 16, 16, 16, 16, 16, 16, None, None)
    assert rc == G.E_NULL
    rc = G.lib().gptl_attention_bwd(1, 64, 128, 4, 1, 0, 16, 16, 16, 16, 16, 16, 20, 16, None)
    assert rc == G.E_ALIGN


def test_clip_and_accumulate_arguments_rejected_without_launch():
    import re
    import os
    hdr = open(os.path.join(G.INCLUDE, "gptlayer.h")).read()
    assert int(re.search(r"#define GPTL_CLIP_WORKSPACE_BYTES (\d+)", hdr).group(1)) == \
        G.CLIP_WORKSPACE_BYTES
    clip = G.lib().adam_step_fp32_master_clip
    ok = (64, 16, 16, 16, 16, 16, 0, 1e-3, 0.9, 0.95, 1e-8, 0.0, 1.0, 16, 16, None)
    for i, bad, code in [(13, None, G.E_NULL),                # no workspace
                         (13, 24, G.E_ALIGN),                 # workspace not 16-byte aligned
                         (12, 0.0, G.E_ARG),                  # max_norm must be positive
                         (12, -1.0, G.E_ARG),
                         (12, float("inf"), G.E_ARG),
                         (12, float("nan"), G.E_ARG),
                         (0, 66, G.E_ARG)]:                   # n % 4 != 0
        args = list(ok)
        args[i] = bad
        assert clip(*args) == code, (i, bad)
    acc = G.lib().gptl_grad_accumulate
    assert acc(64, None, 16, None) == G.E_NULL
    assert acc(64, 16, 20, None) == G.E_ALIGN
    assert acc(66, 16, 1024, None) == G.E_ARG
    assert acc(64, 1024, 1024 + 128, None) == G.E_ARG       # ranges overlap


def test_stack_workspace_and_arguments_rejected_without_launch():
    sh = G.make_shape(2, 64, 128, 4, 512, 2, "fp16")
    saved1, scratch1 = G.workspace_bytes(sh)
    for n in (1, 3, 32):
        saved, scratch = G.stack_workspace_bytes(sh, n)
        per = (saved1 + 255) // 256 * 256
        act = (2 * 64 * 128 * 2 + 255) // 256 * 256
        assert saved == n * per
        assert scratch == (scratch1 + 255) // 256 * 256 + 2 * act
    with pytest.raises(G.GptlError) as e:
        G.stack_workspace_bytes(sh, 0)
    assert e.value.code == G.E_ARG
    w = G.make_weights({n: 4096 for n in G.PARAM_NAMES})
    g = G.make_grads({n: 4096 for n in G.PARAM_NAMES})
    lib = G.lib()
    ws = (G.Weights * 2)(w, w)
    gs = (G.Grads * 2)(g, g)
    assert lib.gpt_stack_fwd(ctypes.byref(sh), 0, ws, 16, 32, 48, None, None) == G.E_ARG
    assert lib.gpt_stack_fwd(ctypes.byref(sh), 2, ws, None, 32, 48, None, None) == G.E_NULL
    assert lib.gpt_stack_fwd(ctypes.byref(sh), 2, ws, 16, 40, 48, None, None) == G.E_ALIGN
    bad = (G.Weights * 2)(w, G.make_weights({n: (8 if n == "w_o" else 4096) for n in G.PARAM_NAMES}))
    assert lib.gpt_stack_fwd(ctypes.byref(sh), 2, bad, 16, 32, 48, None, None) == G.E_ALIGN
    gbad = (G.Grads * 2)(g, G.make_grads({n: (None if n == "b_2" else 4096) for n in G.PARAM_NAMES}))
    assert lib.gpt_stack_bwd(ctypes.byref(sh), 2, ws, 16, 32, 48, 64, 80, gbad, 96, None) == G.E_NULL
    assert lib.gpt_stack_bwd(ctypes.byref(sh), 2, ws, 16, 32, 48, 64, 80, gs, None, None) == G.E_NULL


@pytest.mark.parametrize("shape", [
    dict(batch=1, seq=128, hidden=8192, heads=64, ffn=32768, tp=1, dtype="bf16"),    # h/t = 8192
    dict(batch=1, seq=128, hidden=8192, heads=128, ffn=32768, tp=2, dtype="bf16"),   # 64 heads/shard
    dict(batch=1, seq=2048, hidden=10240, heads=80, ffn=40960, tp=1, dtype="bf16"),
])
def test_wide_shapes_are_accepted(shape):
    """Shapes whose row term covers more than 4096 columns or 32 heads per
    shard are run by the chunked row-dot kernel: sizing accepts them, since
    every launch-time limit is checked up front."""
    saved, scratch = G.workspace_bytes(G.make_shape(**shape))
    assert saved > 0 and scratch > 0


def test_layernorm_backward_limit_is_checked_up_front():
    """hidden 16384 would need 256 KB of running sums per LayerNorm-2
    backward block, above the 227 KB shared-memory limit: the sizing call
    refuses the shape, so fwd / bwd never start a step they cannot finish."""
    sh = G.make_shape(1, 128, 16384, 128, 65536, 1, "bf16")
    with pytest.raises(G.GptlError) as e:
        G.workspace_bytes(sh)
    assert e.value.code == G.E_SHAPE
    w = G.make_weights({n: 4096 for n in G.PARAM_NAMES})
    before = G.launch_count()
    assert G.lib().gpt_layer_fwd(ctypes.byref(sh), ctypes.byref(w), 16, 32, 48, None, None) == G.E_SHAPE
    assert G.launch_count() == before


@pytest.mark.parametrize("name", ["tiny", "gpt2-117m", "large-h10240"])
def test_gelu_recompute_moves_the_activation_to_scratch(name):
    """recompute_gelu keeps A = GeLU(Z) (batch*seq*ffn 16-bit values) out of
    the saved workspace and in scratch; other values of the flag are rejected."""
    c = synth.CONFIGS[name]
    args = (c.batch, c.seq, c.hidden, c.heads, c.ffn, c.tp, c.dtype)
    saved0, scratch0 = G.workspace_bytes(G.make_shape(*args))
    saved1, scratch1 = G.workspace_bytes(G.make_shape(*args, recompute_gelu=1))
    a = c.batch * c.seq * c.ffn * 2
    a256 = (a + 255) // 256 * 256
    assert saved0 - saved1 == a256 and scratch1 - scratch0 == a256
    with pytest.raises(G.GptlError) as e:
        G.workspace_bytes(G.make_shape(*args, recompute_gelu=2))
    assert e.value.code == G.E_SHAPE


def test_weight_copy_arguments_rejected_without_launch():
    """gpt_layer_adam_step / gpt_layer_transpose_weights and the optional
    transposed-weight fields of gptl_weights are checked before any launch."""
    lib = G.lib()
    sh = G.make_shape(2, 64, 128, 4, 512, 2, "fp16")
    st = 16
    args = lambda n_layers, w16t, pre: (ctypes.byref(sh), n_layers, 16, 16, 16, 16, 16, w16t,
                                        1e-3, 0.9, 0.95, 1e-8, 0.0, pre, st, None)
    assert lib.gpt_layer_adam_step(*args(0, 16, 0)) == G.E_ARG
    assert lib.gpt_layer_adam_step(*args(1, 16, 2)) == G.E_ARG
    assert lib.gpt_layer_adam_step(*args(1, None, 0)) == G.E_NULL
    assert lib.gpt_layer_adam_step(*args(1, 24, 1)) == G.E_ALIGN
    assert lib.gpt_layer_transpose_weights(ctypes.byref(sh), 1, None, 16, None) == G.E_NULL
    assert lib.gpt_layer_transpose_weights(ctypes.byref(sh), 0, 16, 16, None) == G.E_ARG
    # the four copies come all together or not at all
    w = G.make_weights({n: 16 for n in G.PARAM_NAMES} | {"w_qkv_t": 16, "w_o_t": 16})
    assert lib.gpt_layer_fwd(ctypes.byref(sh), ctypes.byref(w), 16, 16, 16, None, None) == G.E_NULL
    w = G.make_weights({n: 16 for n in G.PARAM_NAMES} | {n: 16 for n in G.WT_NAMES[:3]} | {"w_2_t": 24})
    assert lib.gpt_layer_fwd(ctypes.byref(sh), ctypes.byref(w), 16, 16, 16, None, None) == G.E_ALIGN
