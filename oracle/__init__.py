"""CPU oracle for one GPT transformer layer's training step.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The CUDA product path never calls it and shares no code with it.

Plain numpy in float64, written from the method the Megatron-LM pages
describe:
  * "Megatron-LM overview" (lshu.cn), §2.2 tensor parallelism, §3.1 mixed
    precision (FP16 matrix math, FP32 master weights, dynamic loss scaling),
    §4.2 the Adam / lr 6e-5 configuration;
  * "Training GPT-2 with Megatron-LM" (devpress.csdn.net), §4.1 the GPT layer
    shapes, §6.2 fused softmax and fused bias-GeLU;
  * "Megatron-LM 3D parallelism" (tbr8.org), §1 column and row splits.

Where the pages are silent (LayerNorm details, GeLU form, biases, mask,
Adam constants, scaler growth rule) the plainest reading is taken and named
in the function that uses it.

Modules:
  layer   layer_fwd / layer_bwd (shard by shard, as the TP split computes it),
          attention_head_fwd / attention_head_bwd (one causal head),
          stack_fwd / stack_bwd (layers of one shape, chained)
  optim   found_inf, adam_step, loss_scale_update, cast_to_16, grad_norm,
          clip_coefficient, accumulate

Parity status: every function is pinned by tests in tests/test_oracle_*.py
(finite differences, sharded == unsharded, closed forms, hand-computed
scaler sequences).  The readings that the pages leave open (GeLU tanh form,
LayerNorm eps, scaler floor and hysteresis, weight decay 0) are fixed by
choice and cannot be pinned to the pages: parity unpinned for those choices
themselves, while the code that implements them is pinned.
"""
from .layer import (layer_fwd, layer_bwd, layer_norm_fwd, layer_norm_bwd, gelu,
                    gelu_prime, causal_softmax, attention_head_fwd, attention_head_bwd,
                    stack_fwd, stack_bwd, STORE_POINTS)
from .optim import (found_inf, adam_step, loss_scale_update, cast_to_16, grad_norm,
                    clip_coefficient, accumulate)

__all__ = ["layer_fwd", "layer_bwd", "stack_fwd", "stack_bwd", "layer_norm_fwd", "layer_norm_bwd", "gelu",
           "gelu_prime", "causal_softmax", "attention_head_fwd", "attention_head_bwd",
           "STORE_POINTS", "found_inf",
           "adam_step", "loss_scale_update", "cast_to_16", "grad_norm", "clip_coefficient",
           "accumulate"]
