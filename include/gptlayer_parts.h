/*
 * gptlayer_parts.h — the building blocks of the layer step, exported one by
 * one so that each kernel can be checked on its own.  Same conventions as
 * gptlayer.h: caller-owned 16-byte-aligned device pointers, asynchronous on
 * `stream`, 0 or a negative GPTL_E_* code, validation before any launch.
 */
#ifndef GPTLAYER_PARTS_H
#define GPTLAYER_PARTS_H

#include "gptlayer.h"

#ifdef __cplusplus
extern "C" {
#endif

/* One operand of gptl_gemm, seen through a 3-D view of a 16-bit tensor:
 * element (x, row, g) lives at ptr + g*g_pitch + row*row_pitch + x
 * (pitches in elements, multiples of 8).
 *   mn_major = 0: `row` indexes M (operand A) or N (operand B) and `x` the
 *                 reduction index k  ("K-major");
 *   mn_major = 1: `row` is k and `x` is the M/N index ("MN-major": the
 *                 tensor core reads it transposed, no copy is made).
 * For group G and k-shard ks the operand's x offset is
 *   (G % x_mod) * x_mul + x_off   and its g coordinate is
 *   G / g_div + (k_shard ? ks : 0).
 * Reads outside the view's extents return zeros. */
typedef struct {
  const void *ptr;
  long long x_ext, rows_ext, g_ext;
  long long row_pitch, g_pitch;
  int mn_major;
  int x_mod, x_mul, x_off;
  int g_div;
  int k_shard;
} gptl_operand;

enum {
  GPTL_ACT_NONE = 0,
  GPTL_ACT_GELU = 1,     /* out = value, out2 = GeLU(value)                   */
  GPTL_ACT_DGELU = 2     /* out = value * GeLU'(aux); out2 (optional) = GeLU(aux) */
};

/* out[G](m, n) = epilogue( sum over ks < k_shards, k < K of A(m,k) * B(n,k) )
 * for m < M, n < N, G < groups, with fp32 accumulation in tensor memory.
 * Output element (m, n) of group G is at
 *   out + (G % o_mod)*o_str_mod + (G / o_mod)*o_str_div + m*ldo + n.
 * Epilogue, in order: + bias[G*bias_g_stride + n] (if bias, 16-bit),
 * + resid[m*ld_resid + n] (if resid; fp32 when resid_f32, else 16-bit), then
 * act: GELU writes the value to out and GeLU(value) to out2; DGELU multiplies
 * by GeLU'(aux at the output's index) and, if out2 is not NULL, also writes
 * GeLU(aux) to out2 (the activation recomputed from its stored argument; with
 * the GELU epilogue's rounding, bit-identical to what GELU wrote for the same
 * 16-bit argument).  out_f32 = 1 stores the fp32 value
 * (act must be GPTL_ACT_NONE); otherwise out is 16-bit, rounded to nearest
 * even.  resid and DGELU do not combine.  Requirements: K % 16 == 0,
 * N % 16 == 0, all offsets/pitches multiples of 8 elements, out (and out2,
 * ws) 16-byte aligned.  The outputs are written by tensor stores of whole
 * 32-row boxes clipped to M x N: nothing outside the M x N window of each
 * group is written, but the groups' windows must not overlap.  causal is
 * reserved and must be 0.
 * Split-K: when out_f32 is set with no bias, resid or act, and ws (16-byte
 * aligned device memory of ws_bytes) is given, the library may cut the K
 * loop of each output tile into slices computed by different SMs; each slice
 * writes fp32 partial sums to ws and a second kernel adds them in slice
 * order (the result is deterministic).  It does so only when the output has
 * too few tiles to fill the GPU and the partials fit in ws_bytes.  ws may be
 * NULL (no split).
 * Column sums: when colsum is not NULL (16-byte aligned fp32 device memory of
 * ceil(M/32) * groups * N floats), the epilogue also writes, for every group
 * G, column n and r < ceil(M/32),
 *   colsum[(r*groups + G)*N + n] = sum over m in [32r, min(32r+32, M)) of
 *                                  out[G](m, n) as stored (16-bit),
 * each added in a fixed order; the caller adds the ceil(M/32) partial rows
 * (a bias gradient).  It needs a 16-bit output (out_f32 = 0) and act other
 * than GELU, and it rules out split-K. */
typedef struct {
  int M, N, K, groups, k_shards, causal;
  gptl_operand a, b;
  void *out;
  int out_f32;
  long long ldo;
  int o_mod;
  long long o_str_mod, o_str_div;
  const void *bias;
  long long bias_g_stride;
  const void *resid;
  long long ld_resid;
  const void *aux;
  void *out2;
  int act;
  int resid_f32;
  void *ws;
  long long ws_bytes;
  float *colsum;
} gptl_gemm_desc;

int gptl_gemm(const gptl_gemm_desc *d, gptl_dtype dtype, gptl_stream_t stream);

/* How gptl_gemm would run *d on the current device (no device work, same
 * argument checks and error codes as gptl_gemm): the tile width bn, the
 * split-K slice count (1 = none) and the use of each SM's two MMA pipelines:
 *   GPTL_GEMM_ALTERNATE  128 x bn tiles alternate between the pipelines;
 *   GPTL_GEMM_K_HALVES   both pipelines on each 128 x bn tile, one half of its
 *                        K range each, summed in a fixed order;
 *   GPTL_GEMM_M256       256 x bn tiles, one 128-row half per pipeline.
 * Results do not depend on the choice beyond fp32 summation order, and are
 * deterministic for a given choice. */
enum { GPTL_GEMM_ALTERNATE = 0, GPTL_GEMM_K_HALVES = 1, GPTL_GEMM_M256 = 2 };
int gptl_gemm_plan(const gptl_gemm_desc *d, gptl_dtype dtype, int *bn, int *split, int *mode);

/* Fused causal attention forward ("Training GPT-2 with Megatron-LM" §6.2
 * fused softmax; scores never leave the chip).  qkv: [tp][batch*seq][3h/tp],
 * shard i's columns [Q_i | K_i | V_i], each head_dim = hidden/heads columns
 * per head.  For every shard, batch element and head:
 *   O = softmax_{q <= p}(Q K^T / sqrt(head_dim)) V   -> o [tp][batch*seq][h/tp]
 *   lse[g][p] = log2 sum_{q <= p} exp2(Q_p.K_q log2(e)/sqrt(head_dim))
 * with g = (shard*batch + batch index)*(heads/tp) + head, lse [g][seq] fp32.
 * head_dim % 16 == 0 and <= 128, seq % 16 == 0. */
int gptl_attention_fwd(int batch, int seq, int hidden, int heads, int tp, gptl_dtype dtype,
                       const void *qkv, void *o, float *lse, gptl_stream_t stream);

/* Fused causal attention backward, the counterpart of gptl_attention_fwd.
 * Given qkv, o and lse of the forward and dout ([tp][batch*seq][h/tp], the
 * gradient with respect to o), writes dQ, dK and dV into the Q, K and V
 * columns of dqkv (same layout as qkv); dvec ([g][seq] fp32, caller scratch)
 * receives D = dO . O per row.  With P = softmax(Q K^T / sqrt(d)) (causal):
 *   dV = P^T dO,  dS = P (dO V^T - D) / sqrt(d),  dQ = dS K,  dK = dS^T Q,
 * P taken in the 16-bit type.  Same size limits as gptl_attention_fwd.
 * dbias (optional, with dbias_part): the QKV bias gradient, [tp][3h/tp] fp32,
 * the column sums of each shard's dqkv over its batch*seq rows, of the values
 * as stored; the kernels that write dQ, dK and dV sum every 32 rows into
 * dbias_part (caller scratch of batch * ceil(seq/32) * 3 * hidden floats) and
 * a second pass adds those in a fixed order.  Both NULL: no bias gradient;
 * only one NULL: GPTL_E_NULL. */
int gptl_attention_bwd(int batch, int seq, int hidden, int heads, int tp, gptl_dtype dtype,
                       const void *qkv, const void *o, const void *dout, const float *lse,
                       float *dvec, void *dqkv, float *dbias_part, float *dbias,
                       gptl_stream_t stream);

/* LayerNorm forward over `rows` rows of width h: y = g*(x-mu)*rstd + b with the
 * biased variance; mu and rstd ([rows] fp32) are saved for the backward.
 * h must split as h/8 = TPR*VPT with TPR a power of two in [16, 256], VPT <= 8. */
int gptl_layernorm_fwd(int rows, int h, gptl_dtype dtype, const void *x, const void *g,
                       const void *b, float eps, void *y, float *mu, float *rstd,
                       gptl_stream_t stream);

/* Scratch bytes gptl_layernorm_bwd needs. */
size_t gptl_layernorm_bwd_scratch_bytes(int rows, int h);

/* LayerNorm backward: dx = resid + LNbwd(gy); dg = sum_rows gy*xhat,
 * db = sum_rows gy (fp32, overwritten); dx_sum (optional, may be NULL) =
 * sum_rows dx.  resid may alias nothing that is written. */
int gptl_layernorm_bwd(int rows, int h, gptl_dtype dtype, const void *gy, const void *x,
                       const float *mu, const float *rstd, const void *g, const void *resid,
                       void *dx, float *dg, float *db, float *dx_sum, void *scratch,
                       gptl_stream_t stream);

/* Scratch bytes gptl_colsum needs. */
size_t gptl_colsum_scratch_bytes(int n, int groups);

/* out[G*n + c] = sum over r < rows of a[G*gstride + r*ld + c] (fp32). */
int gptl_colsum(int rows, int n, int groups, long long ld, long long gstride, gptl_dtype dtype,
                const void *a, float *out, void *scratch, gptl_stream_t stream);

/* The same column sums as gptl_colsum, for callers that cannot hand the
 * library any temporary device memory.  A plug-in or custom operator inside a
 * host framework that owns and pre-plans every device allocation may not call
 * cudaMalloc (nor ask the framework for memory) in the middle of its work, and
 * some deployments forbid device allocation after start-up altogether.  This
 * entry point allocates nothing: its partial sums live in one fixed array of
 * 64 * 16384 floats (4 MiB) in the library's device memory, which every GPU
 * that loads the library holds until the process exits.  (The Megatron-LM
 * pages have no counterpart to this; it is a property of this library.)
 *   - n * groups must be at most 16384, else GPTL_E_TOO_LARGE and nothing is
 *     launched; the other arguments and results are those of gptl_colsum,
 *     summed in the same order.
 *   - The first call on each device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept with the id of the CUDA context it came from: after
 *     a device reset the next call (again outside any capture) looks it up
 *     anew.  Host threads may call concurrently; a mutex guards the lookup.
 *   - All calls share the one array: calls whose kernels may overlap on the
 *     GPU (different streams, or different host threads, on one device) race
 *     and give wrong sums.  Calls in order on one stream are safe.  The array
 *     keeps the last call's partial sums; each call writes every partial it
 *     reads before reading it, so nothing needs clearing in between. */
int gptl_colsum_noalloc(int rows, int n, int groups, long long ld, long long gstride,
                        gptl_dtype dtype, const void *a, float *out, gptl_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* GPTLAYER_PARTS_H */
