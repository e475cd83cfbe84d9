// Stacks of layers of one shape: "Training GPT-2 with Megatron-LM" §4.1
// trains its 2.4B model as --num-layers 32 of them.  The forward runs the
// layers in order, each reading the previous one's output; the backward runs
// them in reverse, each reading the next one's input gradient.  Every layer
// is the single-layer step, so all of its kernels, checks and workspace
// rules carry over; this file only chains the calls and lays out the
// per-layer workspaces.
//
// Included by libgptlayer.cu after gptlayer.cu, in the same translation unit:
// it uses that file's shape check, weight validation and layer_fwd/layer_bwd.
#pragma once

#include <stdint.h>

#include "gptlayer.h"

namespace {

size_t stack_round256(size_t b) { return (b + 255) & ~size_t(255); }

// Per-layer sizes: the saved workspace of one layer (256-byte multiple), the
// shared layer scratch, and one [T, h] 16-bit activation.
struct StackSizes {
  size_t saved, scratch, act;
};

int stack_sizes(const gptl_shape *shape, int n_layers, Dims *D, StackSizes *s) {
  GPTL_TRY(check_shape(shape, D));
  if (n_layers < 1) return GPTL_E_ARG;
  const Ws w = ws_layout(*D);
  s->saved = stack_round256(w.saved);
  s->scratch = stack_round256(w.scratch);
  s->act = (size_t)shape->batch * shape->seq * shape->hidden * 2;
  return GPTL_OK;
}

int validate_grads(const gptl_grads *g) {
  if (!g) return GPTL_E_NULL;
  const float *gp[12] = {g->ln1_g, g->ln1_b, g->w_qkv, g->b_qkv, g->w_o, g->b_o,
                         g->ln2_g, g->ln2_b, g->w_1, g->b_1, g->w_2, g->b_2};
  for (const float *p : gp) {
    if (!p) return GPTL_E_NULL;
    if (!aligned16(p)) return GPTL_E_ALIGN;
  }
  return GPTL_OK;
}

}  // namespace

extern "C" {

int gpt_stack_workspace_bytes(const gptl_shape *shape, int n_layers, size_t *saved_bytes,
                              size_t *scratch_bytes) {
  Dims D;
  StackSizes s;
  GPTL_TRY(stack_sizes(shape, n_layers, &D, &s));
  if (!saved_bytes || !scratch_bytes) return GPTL_E_NULL;
  *saved_bytes = s.saved * (size_t)n_layers;
  *scratch_bytes = s.scratch + 2 * stack_round256(s.act);
  return GPTL_OK;
}

int gpt_stack_fwd(const gptl_shape *shape, int n_layers, const gptl_weights *w, const void *x,
                  void *acts, void *saved, void *scratch, gptl_stream_t stream) {
  Dims D;
  StackSizes s;
  GPTL_TRY(stack_sizes(shape, n_layers, &D, &s));
  if (!w || !x || !acts || !saved || (D.recompute && !scratch)) return GPTL_E_NULL;
  if (!aligned16(x) || !aligned16(acts) || !aligned16(saved) || (scratch && !aligned16(scratch)))
    return GPTL_E_ALIGN;
  for (int l = 0; l < n_layers; ++l) GPTL_TRY(validate_weights(&w[l]));
  GPTL_TRY(device_check());
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const void *in = x;
  for (int l = 0; l < n_layers; ++l) {
    void *out = static_cast<uint8_t *>(acts) + (size_t)l * s.act;
    GPTL_TRY(layer_fwd(D, &w[l], in, out, static_cast<uint8_t *>(saved) + (size_t)l * s.saved,
                       scratch, st));
    in = out;
  }
  return GPTL_OK;
}

int gpt_stack_bwd(const gptl_shape *shape, int n_layers, const gptl_weights *w, const void *x,
                  const void *acts, const void *saved, const void *dy, void *dx,
                  const gptl_grads *g, void *scratch, gptl_stream_t stream) {
  Dims D;
  StackSizes s;
  GPTL_TRY(stack_sizes(shape, n_layers, &D, &s));
  if (!w || !x || !acts || !saved || !dy || !dx || !g || !scratch) return GPTL_E_NULL;
  if (!aligned16(x) || !aligned16(acts) || !aligned16(saved) || !aligned16(dy) ||
      !aligned16(dx) || !aligned16(scratch))
    return GPTL_E_ALIGN;
  for (int l = 0; l < n_layers; ++l) {
    GPTL_TRY(validate_weights(&w[l]));
    GPTL_TRY(validate_grads(&g[l]));
  }
  GPTL_TRY(device_check());
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // input gradients handed between layers alternate between two buffers
  // after the layer scratch, so that no layer reads the buffer it writes
  uint8_t *tmp[2] = {static_cast<uint8_t *>(scratch) + s.scratch,
                     static_cast<uint8_t *>(scratch) + s.scratch + stack_round256(s.act)};
  const void *d = dy;
  for (int l = n_layers - 1; l >= 0; --l) {
    const void *in = l == 0 ? x : static_cast<const uint8_t *>(acts) + (size_t)(l - 1) * s.act;
    void *out = l == 0 ? dx : static_cast<void *>(tmp[l & 1]);
    GPTL_TRY(layer_bwd(D, &w[l], in, static_cast<const uint8_t *>(saved) + (size_t)l * s.saved, d,
                       out, &g[l], scratch, st));
    d = out;
  }
  return GPTL_OK;
}

}  // extern "C"
