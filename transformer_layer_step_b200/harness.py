"""Device memory for one layer's training step, held in torch tensors, and the
four C-ABI calls that make a step.

torch only allocates memory and provides the stream; the fwd, bwd, Adam and
scaler steps all run in libgptlayer.so.  Layout: one flat arena per kind
(16-bit weights, fp32 master / m / v / grad), the 12 parameter tensors at the
offsets the library reports, plus the activation workspace.
"""
from __future__ import annotations

import struct

import numpy as np
import torch

from . import gptlayer as G
from . import synth

TORCH_DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def bits_to_tensor(bits: np.ndarray, dtype: str, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(TORCH_DT[dtype]).to(device)


def tensor_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class LayerStep:
    """Everything one layer step needs on `device`, filled from synth inputs."""

    def __init__(self, cfg: synth.LayerConfig, inputs: dict, device="cuda", hyper=None,
                 recompute_gelu=False, weight_copies=False):
        self.cfg = cfg
        self.hyper = dict(synth.HYPER, **(hyper or {}))
        self.device = torch.device(device)
        self.shape = G.make_shape(cfg.batch, cfg.seq, cfg.hidden, cfg.heads, cfg.ffn, cfg.tp,
                                  cfg.dtype, self.hyper["ln_eps"], recompute_gelu)
        self.offsets, self.n_params = G.param_layout(self.shape)
        saved_b, scratch_b = G.workspace_bytes(self.shape)
        dt = TORCH_DT[cfg.dtype]
        dev = self.device
        T, h = cfg.tokens, cfg.hidden

        # flat parameter arenas
        flat_bits = np.zeros(self.n_params, dtype=np.uint16)
        self.param_shapes = {}
        for name, off in zip(G.PARAM_NAMES, self.offsets):
            arr = inputs["params"][name]
            self.param_shapes[name] = arr.shape
            flat_bits[off:off + arr.size] = arr.reshape(-1)
        self.w16 = bits_to_tensor(flat_bits, cfg.dtype, dev)
        self.master = self.w16.to(torch.float32)       # exact: fp16/bf16 embed in fp32
        self.m = torch.zeros(self.n_params, dtype=torch.float32, device=dev)
        self.v = torch.zeros(self.n_params, dtype=torch.float32, device=dev)
        self.grad = torch.zeros(self.n_params, dtype=torch.float32, device=dev)

        self.x = bits_to_tensor(inputs["x"], cfg.dtype, dev).view(T, h)
        self.y = torch.empty((T, h), dtype=dt, device=dev)
        self.dx = torch.empty((T, h), dtype=dt, device=dev)
        self.dy = torch.zeros((T, h), dtype=dt, device=dev)
        self.saved = torch.empty(max(saved_b, 256), dtype=torch.uint8, device=dev)
        self.scratch = torch.empty(max(scratch_b, 256), dtype=torch.uint8, device=dev)
        self.state = torch.zeros(8, dtype=torch.int32, device=dev)
        self.reset_scaler(self.hyper["init_scale"])

        self.n_layers = 1
        self.w16t = self._weight_copies(weight_copies)
        wp, gp = {}, {}
        for name, off in zip(G.PARAM_NAMES, self.offsets):
            wp[name] = self.w16.data_ptr() + 2 * off
            gp[name] = self.grad.data_ptr() + 4 * off
        wp.update(self._copy_ptrs(0))
        self.weights = G.make_weights(wp)
        self.grads = G.make_grads(gp)

    # ---------------------------------------------------------------- W^T
    def _weight_copies(self, on: bool):
        """With weight_copies the optimizer step (gpt_layer_adam_step) keeps
        transposed copies of the weight matrices in w16t (the same offsets as
        w16), and the backward reads them instead of transposing the weights;
        the first copies are made here."""
        if not on:
            return None
        w16t = torch.zeros_like(self.w16)
        G.transpose_weights(self.shape, self.n_layers, self.w16, w16t, self.stream())
        return w16t

    def _copy_ptrs(self, layer: int) -> dict:
        if self.w16t is None:
            return {}
        base = layer * self.n_layer_params if hasattr(self, "n_layer_params") else 0
        names = dict(zip(G.PARAM_NAMES, self.offsets))
        return {wt: self.w16t.data_ptr() + 2 * (base + names[w])
                for wt, w in zip(G.WT_NAMES, ("w_qkv", "w_o", "w_1", "w_2"))}

    # ---------------------------------------------------------------- state
    def reset_scaler(self, scale: float, tracker: int = 0, step: int = 0):
        words = struct.unpack("<i", struct.pack("<f", scale))[0]
        self.state.copy_(torch.tensor([words, tracker, 0, step, 0, 0, 0, 0], dtype=torch.int32))

    def scaler(self) -> dict:
        s = self.state.cpu().numpy()
        return dict(scale=float(s[:1].view(np.float32)[0]), growth_tracker=int(s[1]),
                    found_inf=int(s[2]), step=int(s[3]))

    def set_dy_bits(self, bits: np.ndarray):
        self.dy.copy_(bits_to_tensor(bits, self.cfg.dtype, self.device).view_as(self.dy))

    # ---------------------------------------------------------------- calls
    def stream(self) -> int:
        return torch.cuda.current_stream(self.device).cuda_stream

    def fwd(self, x=None, y=None):
        G.layer_fwd(self.shape, self.weights, self.x if x is None else x,
                    self.y if y is None else y, self.saved, self.scratch, self.stream())

    def bwd(self, x=None, dy=None, checked=False):
        """gpt_layer_bwd, or with checked=True gpt_layer_bwd_checked (the
        overflow flag set from the gradients as they are written)."""
        x = self.x if x is None else x
        dy = self.dy if dy is None else dy
        if checked:
            G.layer_bwd_checked(self.shape, self.weights, x, self.saved, dy, self.dx, self.grads,
                                self.scratch, self.state, self.stream())
        else:
            G.layer_bwd(self.shape, self.weights, x, self.saved, dy, self.dx, self.grads,
                        self.scratch, self.stream())

    def adam(self, prechecked=False):
        """adam_step_fp32_master (overflow scan + update), or with
        prechecked=True the update alone, on the flag a checked backward set."""
        hp = self.hyper
        if self.w16t is not None:          # also writes the transposed weights
            G.layer_adam_step(self.shape, self.n_layers, self.master, self.m, self.v, self.grad,
                              self.w16, self.w16t, hp["lr"], hp["beta1"], hp["beta2"], hp["eps"],
                              hp["weight_decay"], prechecked, self.state, self.stream())
            return
        fn = G.adam_step_prechecked if prechecked else G.adam_step
        fn(self.n_params, self.master, self.m, self.v, self.grad, self.w16, self.cfg.dtype,
           hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], self.state,
           self.stream())

    def scale_update(self):
        hp = self.hyper
        G.scale_update(self.state, hp["growth_interval"], hp["growth_factor"],
                       hp["backoff_factor"], hp["min_scale"], self.stream())

    def step(self, x=None, dy=None, y=None, fused_check=False):
        """fwd + bwd + Adam + scale update; x, dy and y default to this object's
        buffers (other device buffers of the same shape may be passed).  With
        fused_check the overflow check is folded into the backward
        (gpt_layer_bwd_checked + adam_step_fp32_master_prechecked): the same
        decisions and results, without the pass that re-reads the gradients."""
        self.fwd(x, y)
        self.bwd(x, dy, checked=fused_check)
        self.adam(prechecked=fused_check)
        self.scale_update()

    # ------------------------------------------------------------ readback
    def param_tensor(self, arena: torch.Tensor, name: str) -> torch.Tensor:
        off = self.offsets[G.PARAM_NAMES.index(name)]
        shp = self.param_shapes[name]
        return arena[off:off + int(np.prod(shp))].view(shp)

    def grads_host(self) -> dict:
        return {n: self.param_tensor(self.grad, n).cpu().numpy() for n in G.PARAM_NAMES}

    def params_host_bits(self) -> dict:
        return {n: tensor_to_bits(self.param_tensor(self.w16, n)) for n in G.PARAM_NAMES}


class LayerStack(LayerStep):
    """A stack of layers of one shape on `device` ("Training GPT-2 with
    Megatron-LM" §4.1 trains --num-layers of them): every layer's parameters
    back to back in one flat arena per kind (layer l's block starts at
    l * n_layer_params), the layers' saved workspaces, their outputs `acts`
    ([L, T, h]; the stack's output is acts[-1]), and ONE optimizer step over
    the whole arena.  fwd / bwd make one gpt_stack_fwd / gpt_stack_bwd call;
    adam, scale_update and the scaler helpers are LayerStep's, applied to the
    stack's arenas."""

    def __init__(self, cfg: synth.LayerConfig, layer_params: list, x_bits: np.ndarray,
                 device="cuda", hyper=None, recompute_gelu=False, weight_copies=False):
        self.cfg = cfg
        self.hyper = dict(synth.HYPER, **(hyper or {}))
        self.device = torch.device(device)
        self.shape = G.make_shape(cfg.batch, cfg.seq, cfg.hidden, cfg.heads, cfg.ffn, cfg.tp,
                                  cfg.dtype, self.hyper["ln_eps"], recompute_gelu)
        self.n_layers = L = len(layer_params)
        self.offsets, self.n_layer_params = G.param_layout(self.shape)
        self.n_params = L * self.n_layer_params
        saved_b, scratch_b = G.stack_workspace_bytes(self.shape, L)
        dt = TORCH_DT[cfg.dtype]
        dev = self.device
        T, h = cfg.tokens, cfg.hidden

        flat_bits = np.zeros(self.n_params, dtype=np.uint16)
        self.param_shapes = {}
        for l, params in enumerate(layer_params):
            base = l * self.n_layer_params
            for name, off in zip(G.PARAM_NAMES, self.offsets):
                arr = params[name]
                self.param_shapes[name] = arr.shape
                flat_bits[base + off:base + off + arr.size] = arr.reshape(-1)
        self.w16 = bits_to_tensor(flat_bits, cfg.dtype, dev)
        self.master = self.w16.to(torch.float32)
        self.m = torch.zeros(self.n_params, dtype=torch.float32, device=dev)
        self.v = torch.zeros(self.n_params, dtype=torch.float32, device=dev)
        self.grad = torch.zeros(self.n_params, dtype=torch.float32, device=dev)

        self.x = bits_to_tensor(x_bits, cfg.dtype, dev).view(T, h)
        self.acts = torch.empty((L, T, h), dtype=dt, device=dev)
        self.y = self.acts[L - 1]
        self.dx = torch.empty((T, h), dtype=dt, device=dev)
        self.dy = torch.zeros((T, h), dtype=dt, device=dev)
        self.saved = torch.empty(max(saved_b, 256), dtype=torch.uint8, device=dev)
        self.scratch = torch.empty(max(scratch_b, 256), dtype=torch.uint8, device=dev)
        self.state = torch.zeros(8, dtype=torch.int32, device=dev)
        self.reset_scaler(self.hyper["init_scale"])

        self.w16t = self._weight_copies(weight_copies)
        self.layer_weights, self.layer_grads = [], []
        for l in range(L):
            base = l * self.n_layer_params
            wp = {n: self.w16.data_ptr() + 2 * (base + off) for n, off in zip(G.PARAM_NAMES, self.offsets)}
            wp.update(self._copy_ptrs(l))
            self.layer_weights.append(G.make_weights(wp))
            self.layer_grads.append(G.make_grads(
                {n: self.grad.data_ptr() + 4 * (base + off) for n, off in zip(G.PARAM_NAMES, self.offsets)}))

    def fwd(self, x=None, y=None):
        if y is not None:
            raise ValueError("the stack writes its output into acts[-1]")
        G.stack_fwd(self.shape, self.layer_weights, self.x if x is None else x, self.acts,
                    self.saved, self.scratch, self.stream())

    def bwd(self, x=None, dy=None, checked=False):
        if checked:
            raise ValueError("the stack's backward has no checked variant: scan the arena in Adam")
        G.stack_bwd(self.shape, self.layer_weights, self.x if x is None else x, self.acts,
                    self.saved, self.dy if dy is None else dy, self.dx, self.layer_grads,
                    self.scratch, self.stream())

    def layer_param_tensor(self, arena: torch.Tensor, layer: int, name: str) -> torch.Tensor:
        off = layer * self.n_layer_params + self.offsets[G.PARAM_NAMES.index(name)]
        shp = self.param_shapes[name]
        return arena[off:off + int(np.prod(shp))].view(shp)

    def layer_grads_host(self, layer: int) -> dict:
        return {n: self.layer_param_tensor(self.grad, layer, n).cpu().numpy() for n in G.PARAM_NAMES}

    def param_tensor(self, arena, name):
        raise TypeError("a stack has one block per layer: use layer_param_tensor")
