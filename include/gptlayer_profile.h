/*
 * gptlayer_profile.h — launch accounting and per-launch device timing of
 * the layer-step library, for measurement tools (a benchmark, a profiler
 * front end).  Nothing here changes what the layer computes.
 *
 * Every kernel the library launches is counted.  While a profiling window is
 * open, the library also records a CUDA event on the launch stream when an
 * entry point starts and after each of its kernels, so that each kernel's
 * device duration is the time between two consecutive events on its stream.
 * Each launch carries the kind of kernel and a tag naming the step of the
 * layer it belongs to (the F/B/O step numbering below follows the order of
 * the training step: forward F1..F10, backward B1..B12, optimizer O1..O3).
 *
 * Not thread-safe: open and close a window from the thread that makes the
 * library calls.  The events cost a little device time between launches.
 */
#ifndef GPTLAYER_PROFILE_H
#define GPTLAYER_PROFILE_H

#include "gptlayer.h"

#ifdef __cplusplus
extern "C" {
#endif

/* kernel kinds */
enum {
  GPTL_KIND_GEMM = 0,        /* tcgen05 tensor-core GEMM (every contraction)  */
  GPTL_KIND_LN_FWD = 1,      /* LayerNorm forward                             */
  GPTL_KIND_LN_BWD = 2,      /* LayerNorm backward (rows pass)                */
  GPTL_KIND_RESERVED_3 = 3,  /* not launched (the attention kernels fuse the  */
  GPTL_KIND_RESERVED_4 = 4,  /* scale-mask-softmax)                           */
  GPTL_KIND_COLSUM = 5,      /* column sums (bias gradients), partial pass    */
  GPTL_KIND_REDUCE = 6,      /* final pass of a two-pass column reduction     */
  GPTL_KIND_OVERFLOW = 7,    /* inf/NaN check over the gradient arena         */
  GPTL_KIND_ADAM = 8,        /* fused unscale + Adam + 16-bit cast            */
  GPTL_KIND_SCALE = 9,       /* loss-scale update                             */
  GPTL_KIND_SPLITK = 10,     /* sum of a split-K GEMM's partial tiles         */
  GPTL_KIND_ATTN_FWD = 11,   /* fused causal attention forward                */
  GPTL_KIND_ROWDOT = 12,     /* softmax-backward row term dO . O              */
  GPTL_KIND_TRANSPOSE = 13,  /* token-contiguous copy of a gradient operand   */
  GPTL_KIND_ATTN_BWD = 14,   /* fused causal attention backward (dQ; dK, dV)  */
  GPTL_KIND_CLIP = 15,       /* global-norm clip coefficient (one block)      */
  GPTL_KIND_ACCUMULATE = 16, /* gradient accumulation acc += grad             */
  GPTL_KIND_COUNT = 17
};

/* step tags */
enum {
  GPTL_TAG_NONE = 0,         /* a building-block call made on its own         */
  GPTL_TAG_F1_LN1, GPTL_TAG_F2_QKV, GPTL_TAG_F3_F5_ATTN,
  GPTL_TAG_F6_OUTPROJ, GPTL_TAG_F7_LN2, GPTL_TAG_F8_FFN1_GELU, GPTL_TAG_F10_FFN2,
  GPTL_TAG_B1_B3_DZ, GPTL_TAG_B2_DW2, GPTL_TAG_B2_DB2, GPTL_TAG_B3_DB1, GPTL_TAG_B4_DL2,
  GPTL_TAG_B5_DW1, GPTL_TAG_B6_LN2, GPTL_TAG_B7_DWO, GPTL_TAG_B7_DO, GPTL_TAG_B9_ROWDOT,
  GPTL_TAG_B8_B10_ATTN, GPTL_TAG_B11_DBQKV,
  GPTL_TAG_B11_DWQKV, GPTL_TAG_B11_DL1, GPTL_TAG_B12_LN1,
  GPTL_TAG_O1_OVERFLOW, GPTL_TAG_O2_ADAM, GPTL_TAG_O3_SCALE,
  GPTL_TAG_B2_DOUT_T, GPTL_TAG_B5_L2_T, GPTL_TAG_B7_DH_T, GPTL_TAG_B11_L1_T, GPTL_TAG_B0_WT,
  GPTL_TAG_COUNT
};

typedef struct {
  int kind;   /* GPTL_KIND_*                               */
  int tag;    /* GPTL_TAG_*                                */
  float ms;   /* device duration of the launch, milliseconds */
} gptl_launch_record;

/* Number of kernels this process has launched through the library. */
unsigned long long gptl_launch_count(void);

/* Opens a profiling window able to time `capacity` launches (later launches
 * are counted but not timed).  Creates the CUDA events it needs on the
 * current device.  GPTL_E_ARG if capacity <= 0 or a window is already open;
 * GPTL_E_CUDA if an event cannot be created. */
int gptl_profile_begin(int capacity);

/* Synchronises the device, writes up to `capacity` launch records in launch
 * order to `out`, their number to *n, and the number of launches that ran in
 * the window but were not timed to *dropped; then closes the window and
 * destroys its events.  n and dropped may be NULL.  GPTL_E_ARG if no window
 * is open; GPTL_E_CUDA if the synchronisation or a timing query fails. */
int gptl_profile_end(gptl_launch_record *out, int capacity, int *n, long long *dropped);

/* Short name of a step tag ("F2 qkv", "B9 softmax bwd", ...), static storage. */
const char *gptl_tag_name(int tag);

#ifdef __cplusplus
}
#endif
#endif /* GPTLAYER_PROFILE_H */
