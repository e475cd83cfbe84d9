// gptlayer.cu — the C ABI of the layer-step library: argument validation,
// workspace layout, TMA descriptor encoding, kernel launches.
//
// One GPT layer training step as the Megatron-LM pages describe it
// ("Training GPT-2 with Megatron-LM" §4.1 and §6.2; "Megatron-LM 3D
// parallelism" §1; "Megatron-LM overview" §2.2, §3.1, §4.2), with all
// tensor-parallel shards on one B200.  Every step of the path runs in this
// library's kernels; nothing falls back to the host.
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>

#include "bw_kernels.cuh"
#include "common.cuh"
#include "attn_bwd_tc.cuh"
#include "attn_tc.cuh"
#include "gemm_tc.cuh"
#include "gptlayer_parts.h"
#include "gptlayer_profile.h"

using namespace gptl;

namespace {

#define GPTL_CK(x)                                 \
  do {                                             \
    if ((x) != cudaSuccess) {                      \
      (void)cudaGetLastError();                    \
      return GPTL_E_CUDA;                          \
    }                                              \
  } while (0)
#define GPTL_TRY(x)                                \
  do {                                             \
    const int rc_ = (x);                           \
    if (rc_ != GPTL_OK) return rc_;                \
  } while (0)

constexpr int kMaxDevices = 64;
constexpr int kSmemLimit = 232448;   // 227 KB opt-in dynamic shared memory per block

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ------------------------------------------------------- launch recorder
// Every kernel launch of the library increments g_launches.  While a
// profiling window is open (gptl_profile_begin .. gptl_profile_end) an event
// is also recorded on the launch stream at the start of each entry point and
// after each launch, so that consecutive events bracket one kernel.  The
// tag names the step of the layer the launch belongs to.
struct ProfRec {
  int kind, tag;
  cudaEvent_t a, b;
};
struct Profiler {
  bool on = false;
  cudaEvent_t *pool = nullptr;
  int pool_n = 0, pool_next = 0;
  ProfRec *recs = nullptr;
  int cap = 0, n = 0;
  long long dropped = 0;
  cudaEvent_t prev = nullptr;
};
Profiler g_prof;
int g_tag = GPTL_TAG_NONE;
unsigned long long g_launches = 0;
// While a checked backward runs on this host thread (gpt_layer_bwd_checked),
// the device word that the kernels writing gradients set on an inf or NaN:
// the fp32-output GEMMs, their split-K sums and the column-sum reductions.
thread_local int *g_nonfinite = nullptr;
struct NonfiniteScope {
  int *saved;
  explicit NonfiniteScope(int *f) : saved(g_nonfinite) { g_nonfinite = f; }
  ~NonfiniteScope() { g_nonfinite = saved; }
};

cudaEvent_t prof_event(cudaStream_t st) {
  if (g_prof.pool_next >= g_prof.pool_n) return nullptr;
  cudaEvent_t e = g_prof.pool[g_prof.pool_next];
  if (cudaEventRecord(e, st) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  ++g_prof.pool_next;
  return e;
}

// Marks the start of an entry point's launches on `st`.
void prof_start(cudaStream_t st) {
  if (g_prof.on) g_prof.prev = prof_event(st);
}

// Called after every successful launch on `st`.
void prof_launched(cudaStream_t st, int kind) {
  ++g_launches;
  if (!g_prof.on) return;
  cudaEvent_t e = (g_prof.prev && g_prof.n < g_prof.cap) ? prof_event(st) : nullptr;
  if (!e) {
    ++g_prof.dropped;
    g_prof.prev = nullptr;
    return;
  }
  g_prof.recs[g_prof.n++] = ProfRec{kind, g_tag, g_prof.prev, e};
  g_prof.prev = e;
}

struct TagScope {
  int saved;
  explicit TagScope(int t) : saved(g_tag) { g_tag = t; }
  ~TagScope() { g_tag = saved; }
};

struct DeviceInfo {
  int checked = 0, ok = 0, sms = 0;
};
DeviceInfo g_dev[kMaxDevices];

int device_check(int *sms_out = nullptr) {
  int dev = 0;
  GPTL_CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return GPTL_E_ARCH;
  DeviceInfo &d = g_dev[dev];
  if (!d.checked) {
    int major = 0, sms = 0;
    GPTL_CK(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    GPTL_CK(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    d.ok = (major == 10);
    d.sms = sms;
    d.checked = 1;
  }
  if (!d.ok) return GPTL_E_ARCH;
  if (sms_out) *sms_out = d.sms;
  return GPTL_OK;
}

// ------------------------------------------------------------ TMA encoding
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

int mn_chunk_width(long long rows_tile) {
  return rows_tile % 64 == 0 ? 64 : (rows_tile % 32 == 0 ? 32 : 16);
}

int encode_operand(CUtensorMap *map, const gptl_operand &o, gptl_dtype dt, int rows_tile, int w) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return GPTL_E_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)o.x_ext, (cuuint64_t)o.rows_ext, (cuuint64_t)o.g_ext};
  cuuint64_t strides[2] = {(cuuint64_t)o.row_pitch * 2,
                           (cuuint64_t)(o.g_ext > 1 ? o.g_pitch : o.rows_ext * o.row_pitch) * 2};
  cuuint32_t box[3], es[3] = {1, 1, 1};
  CUtensorMapSwizzle swz;
  if (!o.mn_major) {
    box[0] = 64;
    box[1] = (cuuint32_t)rows_tile;
    box[2] = 1;
    swz = CU_TENSOR_MAP_SWIZZLE_128B;
  } else {
    box[0] = (cuuint32_t)w;
    box[1] = (cuuint32_t)kBK;
    box[2] = 1;
    swz = w == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                  : (w == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  }
  const CUresult r =
      fn(map, dt == GPTL_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
         const_cast<void *>(o.ptr), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GPTL_OK : GPTL_E_CUDA;
}

// Tensor map of a GEMM output for the epilogue's 32-row x 64-byte store
// boxes (64B swizzle).  Group G of the output sits at
// (G % o_mod) * str_mod + (G / o_mod) * str_div elements; flat = 1 maps it as
// one coordinate z = G (str_div apart), else as (z, w) = (G % o_mod, G / o_mod).
int encode_output(CUtensorMap *map, void *ptr, int f32, gptl_dtype dt, long long N, long long M,
                  long long ld, int groups, int o_mod, long long str_mod, long long str_div,
                  int *flat) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return GPTL_E_CUDA;
  const long long es = f32 ? 4 : 2;
  cuuint64_t dims[4], strides[3];
  dims[0] = (cuuint64_t)N;
  dims[1] = (cuuint64_t)M;
  strides[0] = (cuuint64_t)(ld * es);
  const long long plane = ld * M * es;   // a valid stride for an extent-1 dimension
  if (o_mod == 1 || groups == 1) {
    *flat = 1;
    dims[2] = (cuuint64_t)groups;
    dims[3] = 1;
    const long long s2 = (o_mod == 1 ? str_div : str_mod) * es;
    strides[1] = (cuuint64_t)(groups > 1 ? s2 : plane);
    strides[2] = (cuuint64_t)(groups > 1 ? s2 * groups : plane);
  } else {
    *flat = 0;
    const long long nd = (groups + o_mod - 1) / o_mod;
    dims[2] = (cuuint64_t)o_mod;
    dims[3] = (cuuint64_t)nd;
    strides[1] = (cuuint64_t)(str_mod * es);
    strides[2] = (cuuint64_t)(nd > 1 ? str_div * es : str_mod * es * o_mod);
  }
  for (int i = 0; i < 3; ++i)
    if (strides[i] == 0 || strides[i] % 16 || strides[i] >= (1ull << 40)) return GPTL_E_SHAPE;
  cuuint32_t box[4] = {(cuuint32_t)(64 / es), 32, 1, 1}, ones[4] = {1, 1, 1, 1};
  const CUtensorMapDataType ty = f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                     : (dt == GPTL_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                        : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16);
  const CUresult r = fn(map, ty, 4, ptr, dims, strides, box, ones, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? GPTL_OK : GPTL_E_CUDA;
}

int check_operand(const gptl_operand &o) {
  if (!o.ptr) return GPTL_E_NULL;
  if (!aligned16(o.ptr)) return GPTL_E_ALIGN;
  if (o.x_ext <= 0 || o.rows_ext <= 0 || o.g_ext <= 0 || o.row_pitch <= 0) return GPTL_E_SHAPE;
  if (o.row_pitch % 8 || (o.g_ext > 1 && (o.g_pitch <= 0 || o.g_pitch % 8))) return GPTL_E_SHAPE;
  if (o.x_mod < 1 || o.g_div < 1 || o.x_mul % 8 || o.x_off % 8 || o.x_mul < 0 || o.x_off < 0)
    return GPTL_E_SHAPE;
  if (o.x_ext >= (1ll << 32) || o.rows_ext >= (1ll << 32) || o.g_ext >= (1ll << 32))
    return GPTL_E_SHAPE;
  return GPTL_OK;
}

int pick_bn(const gptl_gemm_desc &d, int sms) {
  if (d.N <= 256) return d.N;
  const long long m_tiles = (d.M + kBM - 1) / kBM;
  long long best_cost = -1;
  int best = 256;
  for (int bn : {256, 128}) {
    const long long tiles = m_tiles * ((d.N + bn - 1) / bn) * d.groups;
    const long long waves = (tiles + sms - 1) / sms;
    const long long cost = waves * (bn + 64);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

// Tiling of one GEMM call: BN, split-K slices (fp32 output with a workspace
// only) and the use of the CTA's two pipelines, chosen by a time estimate in
// microseconds.  Per-k-block times measured on B200 (BN = 256; a k-block is
// 64 deep), with both pipelines of an SM busy unless noted:
//   alternate   tiles alternate between the pipelines, 128 x BN tiles:
//               1.17 per k-block of each pipeline (0.9 when one runs alone);
//               one tile's epilogue overlaps the other pipeline's MMAs
//   K halves    both pipelines on one 128 x BN tile: 1.13 per k-block of each
//   m2          256 x BN tiles, one M half per pipeline, one shared ring:
//               0.8 per k-block of the pair (a third less operand traffic
//               from L2 per FLOP than 128 x BN tiles)
// Narrower tiles (BN 224, 192, 160, 128) take proportionally less: half of
// the time scales with the MMA work (BN) and half with the operand bytes
// (rows of A + BN).  They trade a little of that rate for a tile count that
// fills the last wave: a 2048 x 10240 output is 320 tiles of 256 x 256 (2.2
// waves of 148 SMs, so three rounds at 72 % occupancy) but 432 tiles of
// 256 x 192 (2.9 waves, 97 %).
// The K-halves and m2 modes cannot overlap a tile's epilogue with the next
// tile's MMAs (all 512 TMEM columns hold the tile): ~1.3 us per 128 x 256
// half tile, ~5 with GeLU / GeLU' (measured: the 256-row mode loses to
// alternating tiles on the GeLU GEMMs, wins on the others).  Split-K adds the
// partial-sum pass, (2 split + 1) fp32 arrays at ~4 TB/s plus a launch.
struct GemmTiling {
  int bn, split, pipe_k, m2;
};
GemmTiling choose_tiling(const gptl_gemm_desc &d, int sms, bool can_split) {
  GemmTiling best{pick_bn(d, sms), 1, 0, 0};
  const long long kb_all = (long long)((d.K + kBK - 1) / kBK) * d.k_shards;
  const double out_bytes = (double)d.groups * d.M * d.N * 4.0;
  const double e_half = (d.act == GPTL_ACT_NONE ? 1.3 : 5.0);
  double best_t = -1.0;
  static const int kBnChoices[] = {256, 224, 192, 160, 128};
  for (int bn_c : kBnChoices) {
    const int bn = d.N <= 256 ? d.N : bn_c;
    if (d.N <= 256 && bn_c != 256) break;         // N fits one tile column: BN = N
    const double e_tile = e_half * bn / 256.0;
    const long long n_tiles = (d.N + bn - 1) / bn;
    for (int mode = 0; mode < 3; ++mode) {          // alternate, K halves, m2
      if (mode == 2 && d.M <= kBM) continue;
      const int rows = mode == 2 ? 2 * kBM : kBM;
      const long long m_tiles = (d.M + rows - 1) / rows;
      const long long tiles = m_tiles * n_tiles * d.groups;
      // per-k-block time of this BN: half scales with BN, half with A rows + BN
      const double width = 0.5 * bn / 256.0 + 0.5 * (double)(rows + bn) / (double)(rows + 256);
      for (int sp = 1; sp <= (can_split ? 8 : 1); ++sp) {
        if (sp > (d.K + kBK - 1) / kBK) break;
        if (sp > 1 && (double)sp * out_bytes > (double)d.ws_bytes) break;
        // K halves: every slice must give each pipeline at least one k-block
        if (mode == 1 && ((d.K + kBK - 1) / kBK) / sp < 2) continue;
        const long long items = tiles * sp;
        const long long kb = (kb_all + sp - 1) / sp;
        const long long per_cta = (items + sms - 1) / sms;
        double t;
        if (mode == 0)
          t = per_cta >= 2 ? (double)((per_cta + 1) / 2) * kb * 1.17 * width + e_tile
                           : kb * 0.9 * width + e_tile;
        else if (mode == 1)
          t = (double)per_cta * ((kb + 1) / 2 * 1.13 * width + e_tile);
        else
          t = (double)per_cta * (kb * 0.8 * width + 2.0 * e_tile);
        if (sp > 1) t += (2.0 * sp + 1.0) * out_bytes / 4.0e6 + 3.0;
        if (best_t < 0 || t < best_t * 0.999) {
          best_t = t;
          best = GemmTiling{bn, sp, mode == 1 ? 1 : 0, mode == 2 ? 1 : 0};
        }
      }
    }
  }
  return best;
}

template <typename T>
int launch_gemm_t(const GemmParams &p, int grid, int smem, cudaStream_t stream) {
  // opt-ins per device, for the instantiations without and with column sums
  static bool attr_set[kMaxDevices][2] = {};
  int dev = 0;
  GPTL_CK(cudaGetDevice(&dev));
  const int cs = p.colsum ? 1 : 0;
  auto kern = cs ? gemm_tc_kernel<T, true> : gemm_tc_kernel<T, false>;
  if (!attr_set[dev][cs]) {
    // the kernel splits its registers by role (setmaxnreg), a split that
    // adds up only when every thread was launched with kGemmRegs
    cudaFuncAttributes fa{};
    GPTL_CK(cudaFuncGetAttributes(&fa, kern));
    if (fa.numRegs != kGemmRegs || fa.maxThreadsPerBlock < kGemmThreads) return GPTL_E_CUDA;
    GPTL_CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
    attr_set[dev][cs] = true;
  }
  kern<<<grid, kGemmThreads, smem, stream>>>(p);
  GPTL_CK(cudaGetLastError());
  prof_launched(stream, GPTL_KIND_GEMM);
  return GPTL_OK;
}

// Argument checks of gptl_gemm (no device work).
int gemm_validate(const gptl_gemm_desc &d, gptl_dtype dt) {
  if (dt != GPTL_FP16 && dt != GPTL_BF16) return GPTL_E_DTYPE;
  if (!d.out) return GPTL_E_NULL;
  if (!aligned16(d.out)) return GPTL_E_ALIGN;
  if (d.M <= 0 || d.N <= 0 || d.K <= 0 || d.groups <= 0 || d.k_shards <= 0) return GPTL_E_SHAPE;
  if (d.K % 16 || d.N % 16 || d.causal != 0 || d.o_mod < 1) return GPTL_E_SHAPE;
  const int oal = d.out_f32 ? 4 : 8;
  if (d.ldo % oal || d.o_str_mod % oal || d.o_str_div % oal || d.ldo < d.N) return GPTL_E_SHAPE;
  if (d.bias && (!aligned16(d.bias) || d.bias_g_stride % 8)) return GPTL_E_ALIGN;
  if (d.resid && (!aligned16(d.resid) || d.ld_resid % 8)) return GPTL_E_ALIGN;
  if (d.act == GPTL_ACT_GELU && !d.out2) return GPTL_E_NULL;
  if (d.act == GPTL_ACT_DGELU && !d.aux) return GPTL_E_NULL;
  if ((d.out2 && !aligned16(d.out2)) || (d.aux && !aligned16(d.aux))) return GPTL_E_ALIGN;
  if (d.act < 0 || d.act > 2 || (d.out_f32 && d.act != GPTL_ACT_NONE)) return GPTL_E_SHAPE;
  if (d.resid && d.act == GPTL_ACT_DGELU) return GPTL_E_SHAPE;   // one epilogue input per GEMM
  if (d.colsum && !aligned16(d.colsum)) return GPTL_E_ALIGN;
  if (d.colsum && (d.out_f32 || d.act == GPTL_ACT_GELU)) return GPTL_E_SHAPE;
  GPTL_TRY(check_operand(d.a));
  GPTL_TRY(check_operand(d.b));
  return GPTL_OK;
}

GemmTiling gemm_plan(const gptl_gemm_desc &d, int sms) {
  const bool can_split = d.out_f32 && !d.bias && !d.resid && d.act == GPTL_ACT_NONE && d.ws &&
                         aligned16(d.ws) && !d.colsum;
  return choose_tiling(d, sms, can_split);
}

int run_gemm(const gptl_gemm_desc &d, gptl_dtype dt, cudaStream_t stream) {
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  GPTL_TRY(gemm_validate(d, dt));
  GemmParams p;
  memset(&p, 0, sizeof(p));
  const GemmTiling tl = gemm_plan(d, sms);
  const int bn = tl.bn;
  const int wa = d.a.mn_major ? mn_chunk_width(kBM) : 64;
  const int wb = d.b.mn_major ? mn_chunk_width(bn) : 64;
  const int a_rows = tl.m2 ? 2 * kBM : kBM;   // rows of A per tile
  GPTL_TRY(encode_operand(&p.map_a, d.a, dt, a_rows, wa));
  GPTL_TRY(encode_operand(&p.map_b, d.b, dt, bn, wb));
  auto rule = [](const gptl_operand &o, int w) {
    OperandRule r;
    r.mn_major = o.mn_major;
    r.w = w;
    r.x_mod = o.x_mod;
    r.x_mul = o.x_mul;
    r.x_off = o.x_off;
    r.g_div = o.g_div;
    r.k_shard = o.k_shard;
    return r;
  };
  p.ra = rule(d.a, wa);
  p.rb = rule(d.b, wb);
  p.M = d.M;
  p.N = d.N;
  p.K = d.K;
  p.groups = d.groups;
  p.k_shards = d.k_shards;
  p.bn = bn;
  int bn_alloc = 32;
  while (bn_alloc < bn) bn_alloc *= 2;
  p.bn_alloc = bn_alloc;
  p.tmem_cols = 2 * bn_alloc;
  const int stage_bytes = (a_rows + bn) * kBK * 2;
  // stages per ring: two rings (one per pipeline), or one shared ring in m2
  const int rings = tl.m2 ? 1 : 2;
  p.stages = (kSmemLimit - 2048 - kStagingBytes) / (rings * stage_bytes);
  if (p.stages > 4) p.stages = 4;
  if (p.stages < 2) return GPTL_E_SHAPE;
  const int smem = 1024 + rings * p.stages * stage_bytes + kStagingBytes + 512;
  const uint32_t fmt = dt == GPTL_BF16 ? 1u : 0u;
  p.idesc = (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)d.a.mn_major << 15) |
            ((uint32_t)d.b.mn_major << 16) | ((uint32_t)(bn >> 3) << 17) |
            ((uint32_t)(kBM >> 4) << 24);
  p.m_tiles = (d.M + a_rows - 1) / a_rows;
  p.n_tiles = (d.N + bn - 1) / bn;
  const long long tiles = (long long)p.m_tiles * p.n_tiles * d.groups;
  p.split = tl.split;
  p.pipe_k = tl.pipe_k;
  p.m2 = tl.m2;
  p.ws = static_cast<float *>(d.ws);
  p.ws_slice = (long long)d.groups * d.M * d.N;
  p.total_tiles = tiles * p.split;
  {  // a band of N tiles per wave: every M tile of the band runs at once
    long long band = sms / p.m_tiles;
    if (band < 1) band = 1;
    if (band > p.n_tiles) band = p.n_tiles;
    p.band = (int)band;
  }
  if (p.split > 1) {            // partials [split * groups][M][N], dense fp32
    int flat = 1;
    GPTL_TRY(encode_output(&p.map_o, d.ws, 1, dt, d.N, d.M, d.N, p.split * d.groups, 1, 0,
                           (long long)d.M * d.N, &flat));
    p.o_flat = 1;
  } else {
    GPTL_TRY(encode_output(&p.map_o, d.out, d.out_f32, dt, d.N, d.M, d.ldo, d.groups, d.o_mod,
                           d.o_str_mod, d.o_str_div, &p.o_flat));
    if (d.act == GPTL_ACT_GELU || (d.act == GPTL_ACT_DGELU && d.out2)) {
      p.write_o2 = 1;
      int flat2 = 0;
      GPTL_TRY(encode_output(&p.map_o2, d.out2, 0, dt, d.N, d.M, d.ldo, d.groups, d.o_mod,
                             d.o_str_mod, d.o_str_div, &flat2));
    }
  }
  p.ldo = d.ldo;
  p.o_mod = d.o_mod;
  p.o_str_mod = d.o_str_mod;
  p.o_str_div = d.o_str_div;
  p.out_f32 = d.out_f32;
  p.bias = d.bias;
  p.bias_g_stride = d.bias_g_stride;
  p.resid = d.resid;
  p.resid_f32 = d.resid_f32 ? 1 : 0;
  p.ld_resid = d.ld_resid;
  p.aux = d.aux;
  p.act = d.act;
  p.nonfinite = d.out_f32 ? g_nonfinite : nullptr;
  p.colsum = d.colsum;
  p.colsum_rows = (d.M + 31) / 32;
  // fp32 outputs without a residual are weight gradients, which the next
  // kernels do not read: their stores leave L2 first instead of evicting
  // the operands that the other CTAs are still reading
  p.out_evict_first = d.out_f32 && !d.resid && p.split == 1;
  const int grid = (int)(p.total_tiles < sms ? p.total_tiles : sms);
  if (dt == GPTL_FP16) GPTL_TRY(launch_gemm_t<__half>(p, grid, smem, stream));
  else GPTL_TRY(launch_gemm_t<__nv_bfloat16>(p, grid, smem, stream));
  if (p.split > 1) {
    const long long n4 = p.ws_slice / 4;
    long long blocks = (n4 + 255) / 256;
    if (blocks > 8 * sms) blocks = 8 * sms;
    splitk_reduce_kernel<<<(unsigned)blocks, 256, 0, stream>>>(
        p.ws, p.ws_slice, p.split, d.M, d.N, d.groups, static_cast<float *>(d.out), d.ldo,
        d.o_mod, d.o_str_mod, d.o_str_div, p.nonfinite);
    GPTL_CK(cudaGetLastError());
    prof_launched(stream, GPTL_KIND_SPLITK);
  }
  return GPTL_OK;
}

// ------------------------------------------------------------- attention
// Fused causal attention forward over the QKV buffer C [t][T][3h/t] (shard
// columns [Q_i | K_i | V_i], head-major): O [t][T][h/t] and the base-2
// log-sum-exp of every row's scaled scores, lse [t*b*(a/t)][s].
int run_attn_fwd(int b, int s, int hs, int as, int t, int d, gptl_dtype dt, const void *c, void *o,
                 float *lse, cudaStream_t st) {
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  if (d % 16 || d > 128 || hs % 8 || s <= 0 || s % 16 || as <= 0 || b <= 0 || t <= 0)
    return GPTL_E_SHAPE;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return GPTL_E_CUDA;
  AttnParams p;
  memset(&p, 0, sizeof(p));
  const CUtensorMapDataType ty =
      dt == GPTL_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t dims[3] = {(cuuint64_t)(3 * hs), (cuuint64_t)s, (cuuint64_t)t * b};
  cuuint64_t strides[2] = {(cuuint64_t)3 * hs * 2, (cuuint64_t)s * 3 * hs * 2};
  cuuint32_t es[3] = {1, 1, 1};
  cuuint32_t box_qk[3] = {16, 128, 1};
  if (fn(&p.map_qk, ty, 3, const_cast<void *>(c), dims, strides, box_qk, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GPTL_E_CUDA;
  const int vw = d % 64 == 0 ? 64 : (d % 32 == 0 ? 32 : 16);
  cuuint32_t box_v[3] = {(cuuint32_t)vw, 64, 1};
  const CUtensorMapSwizzle vsw = vw == 64 ? CU_TENSOR_MAP_SWIZZLE_128B
                                          : (vw == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  if (fn(&p.map_v, ty, 3, const_cast<void *>(c), dims, strides, box_v, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, vsw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return GPTL_E_CUDA;
  p.s = s; p.d = d; p.hs = hs; p.as = as;
  p.groups = t * b * as;
  p.q_tiles = (s + kAttnTile - 1) / kAttnTile;
  p.vw = vw;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)d);
  const uint32_t fmt = dt == GPTL_BF16 ? 1u : 0u;
  p.idesc_s = (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(kAttnTile >> 3) << 17) |
              ((uint32_t)(kAttnTile >> 4) << 24);
  p.idesc_pv = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 16) | ((uint32_t)(d >> 3) << 17) |
               ((uint32_t)(kAttnTile >> 4) << 24);
  p.o = o;
  p.lse = lse;
  p.items = (long long)p.groups * p.q_tiles;
  p.q_off = 0; p.k_off = hs; p.v_off = 2 * hs;
  // P 2 x 32 KB, Q, the K / V ring (as deep as fits, 2..4 stages), barriers
  // and the half-row lse; at least 120 KB so that one CTA (and its 512
  // tensor-memory columns) owns each SM
  const int kv_stage = 2 * 128 * d * 2;
  p.kv_stages = (kSmemLimit - 1024 - 65536 - 128 * d * 2 - kAttnTailBytes) / kv_stage;
  if (p.kv_stages > 4) p.kv_stages = 4;
  if (p.kv_stages < 2) return GPTL_E_SHAPE;
  int smem = 1024 + 65536 + 128 * d * 2 + p.kv_stages * kv_stage + kAttnTailBytes;
  if (smem < 120 * 1024) smem = 120 * 1024;
  const int grid = (int)(p.items < sms ? p.items : sms);
  // the shared-memory opt-in is recorded per device and per dtype (both
  // instantiations have the same function-pointer type)
  static bool attr_set[kMaxDevices][2] = {};
  int dev = 0;
  GPTL_CK(cudaGetDevice(&dev));
  auto launch = [&](auto kern) -> int {
    if (!attr_set[dev][dt]) {
      GPTL_CK(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
      attr_set[dev][dt] = true;
    }
    kern<<<grid, kAttnThreads, smem, st>>>(p);
    GPTL_CK(cudaGetLastError());
    return GPTL_OK;
  };
  if (dt == GPTL_FP16) GPTL_TRY(launch(attn_fwd_kernel<__half>));
  else GPTL_TRY(launch(attn_fwd_kernel<__nv_bfloat16>));
  prof_launched(st, GPTL_KIND_ATTN_FWD);
  return GPTL_OK;
}

// Fused causal attention backward: dQ, dK, dV into the Q, K, V columns of
// dC [t][T][3h/t] from C, dO [t][T][h/t], the forward's row log-sum-exp and
// D = dO . O.  Two kernels (per query block: dQ; per key block: dK, dV).
// part (may be null): the bias-gradient partials of dC, [b * ceil(s/32)][t * 3hs] fp32.
int run_attn_bwd(int b, int s, int hs, int as, int t, int d, gptl_dtype dt, const void *c,
                 const void *dout, const float *lse, const float *dvec, void *dc, float *part,
                 cudaStream_t st) {
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  if (d % 16 || d > 128 || hs % 8 || s <= 0 || s % 16 || as <= 0 || b <= 0 || t <= 0)
    return GPTL_E_SHAPE;
  EncodeTiledFn fn = encode_fn();
  if (!fn) return GPTL_E_CUDA;
  AttnBwdParams p;
  memset(&p, 0, sizeof(p));
  const CUtensorMapDataType ty =
      dt == GPTL_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint32_t es[3] = {1, 1, 1}, box[3] = {16, 128, 1};
  {
    cuuint64_t dims[3] = {(cuuint64_t)(3 * hs), (cuuint64_t)s, (cuuint64_t)t * b};
    cuuint64_t strides[2] = {(cuuint64_t)3 * hs * 2, (cuuint64_t)s * 3 * hs * 2};
    if (fn(&p.map_c, ty, 3, const_cast<void *>(c), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
           CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTL_E_CUDA;
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)hs, (cuuint64_t)s, (cuuint64_t)t * b};
    cuuint64_t strides[2] = {(cuuint64_t)hs * 2, (cuuint64_t)s * hs * 2};
    if (fn(&p.map_do, ty, 3, const_cast<void *>(dout), dims, strides, box, es,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return GPTL_E_CUDA;
  }
  p.s = s; p.d = d; p.hs = hs; p.as = as;
  p.groups = t * b * as;
  p.tiles = (s + 127) / 128;
  p.scale = 1.0f / sqrtf((float)d);
  p.scale_log2 = 1.4426950408889634f * p.scale;
  const uint32_t fmt = dt == GPTL_BF16 ? 1u : 0u;
  p.idesc_s = (1u << 4) | (fmt << 7) | (fmt << 10) | (16u << 17) | (8u << 24);
  p.idesc_acc = (1u << 4) | (fmt << 7) | (fmt << 10) | (1u << 16) | ((uint32_t)(d >> 3) << 17) | (8u << 24);
  p.lse = lse;
  p.dvec = dvec;
  p.dc = dc;
  p.items = (long long)p.groups * p.tiles;
  p.q_off = 0; p.k_off = hs; p.v_off = 2 * hs;
  p.colsum = part;
  p.batch = b;
  p.cs_rows = (s + 31) / 32;
  p.cs_width = t * 3 * hs;
  const int tb = 256 * d;
  // rings as deep as shared memory allows (up to 4 stages): dQ kernel dS
  // 32 KB + Q, dO + K/V stages; dK/dV kernel P^T, dS^T 64 KB + K, V + Q/dO
  // stages + the staged lse / D vectors
  int nkv = (kSmemLimit - 1024 - 32768 - 2 * tb - 512) / (2 * tb);
  if (nkv > 4) nkv = 4;
  if (nkv < 2) return GPTL_E_SHAPE;
  int smem_dq = 1024 + 32768 + 2 * tb + nkv * 2 * tb + 512;
  int nst = (kSmemLimit - 1024 - 65536 - 2 * tb - 2048 - 512) / (2 * tb);
  if (nst > 4) nst = 4;
  if (nst < 1) return GPTL_E_SHAPE;
  int smem_kv = 1024 + 65536 + 2 * tb + nst * 2 * tb + 2048 + 512;
  p.kv_stages = nkv;
  p.qdo_stages = nst;
  // at least 120 KB: one CTA (and its 512 tensor-memory columns) per SM
  if (smem_dq < 120 * 1024) smem_dq = 120 * 1024;
  if (smem_kv < 120 * 1024) smem_kv = 120 * 1024;
  if (smem_dq > kSmemLimit || smem_kv > kSmemLimit) return GPTL_E_SHAPE;
  const int grid = (int)(p.items < sms ? p.items : sms);
  static bool attr_set[kMaxDevices][2] = {};
  int dev = 0;
  GPTL_CK(cudaGetDevice(&dev));
  auto launch = [&](auto kq, auto kkv) -> int {
    if (!attr_set[dev][dt]) {
      GPTL_CK(cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
      GPTL_CK(cudaFuncSetAttribute(kkv, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit));
      attr_set[dev][dt] = true;
    }
    kq<<<grid, kAttnBwdThreads, smem_dq, st>>>(p);
    GPTL_CK(cudaGetLastError());
    prof_launched(st, GPTL_KIND_ATTN_BWD);
    kkv<<<grid, kAttnBwdThreads, smem_kv, st>>>(p);
    GPTL_CK(cudaGetLastError());
    prof_launched(st, GPTL_KIND_ATTN_BWD);
    return GPTL_OK;
  };
  if (dt == GPTL_FP16) return launch(attn_bwd_dq_kernel<__half>, attn_bwd_kv_kernel<__half>);
  return launch(attn_bwd_dq_kernel<__nv_bfloat16>, attn_bwd_kv_kernel<__nv_bfloat16>);
}

// out [cols][rows] = in [rows][cols]^T (16-bit), for `batch` matrices
// `bs_in` / `bs_out` elements apart.
// One launch for up to kMaxTransposeJobs transposes (see transpose16_kernel).
struct TransposeSpec {
  int rows, cols;
  const void *in;
  long long ld_in;
  void *out;
  long long ld_out;
  int batch;
  long long bs_in, bs_out;
};
int run_transposes(const TransposeSpec *spec, int n, cudaStream_t st) {
  if (n < 1 || n > kMaxTransposeJobs) return GPTL_E_ARG;
  TransposeJobs jobs;
  memset(&jobs, 0, sizeof(jobs));
  long long tiles = 0;
  for (int i = 0; i < n; ++i) {
    const TransposeSpec &s = spec[i];
    if (s.rows <= 0 || s.cols <= 0 || s.rows % 8 || s.cols % 8 || s.ld_in % 8 || s.ld_out % 8 ||
        s.batch < 1 || s.bs_in % 8 || s.bs_out % 8)
      return GPTL_E_SHAPE;
    TransposeJob &J = jobs.job[i];
    J.in = static_cast<const uint16_t *>(s.in);
    J.out = static_cast<uint16_t *>(s.out);
    J.rows = s.rows;
    J.cols = s.cols;
    J.ld_in = s.ld_in;
    J.ld_out = s.ld_out;
    J.bs_in = s.bs_in;
    J.bs_out = s.bs_out;
    J.tiles_c = (s.cols + 63) / 64;
    J.tiles_r = (s.rows + 63) / 64;
    J.tile0 = tiles;
    tiles += (long long)J.tiles_c * J.tiles_r * s.batch;
  }
  jobs.n = n;
  if (tiles >= (1ll << 31)) return GPTL_E_SHAPE;
  transpose16_kernel<<<(unsigned)tiles, 256, 0, st>>>(jobs);
  GPTL_CK(cudaGetLastError());
  prof_launched(st, GPTL_KIND_TRANSPOSE);
  return GPTL_OK;
}

int run_transpose(int rows, int cols, const void *in, long long ld_in, void *out, long long ld_out,
                  cudaStream_t st, int batch = 1, long long bs_in = 0, long long bs_out = 0) {
  const TransposeSpec s{rows, cols, in, ld_in, out, ld_out, batch, bs_in, bs_out};
  return run_transposes(&s, 1, st);
}

// D[g][p] = dO_p . O_p over each head's columns (the softmax backward's row term).
int run_attn_rowdot(long long rows, int s, int hs, int as, int d, gptl_dtype dt, const void *dout,
                    const void *o, float *dvec, cudaStream_t st) {
  if (hs % 8 || d % 8 || d <= 0 || d / 8 > kRowdotChunkVec || (long long)as * d != hs) return GPTL_E_SHAPE;
  const unsigned grid = (unsigned)((rows + 7) / 8);
  if (dt == GPTL_FP16)
    attn_rowdot_kernel<__half><<<grid, 256, 0, st>>>((const __half *)dout, (const __half *)o, dvec,
                                                     rows, s, hs, as, d);
  else
    attn_rowdot_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16 *)dout, (const __nv_bfloat16 *)o, dvec, rows, s, hs, as, d);
  GPTL_CK(cudaGetLastError());
  prof_launched(st, GPTL_KIND_ROWDOT);
  return GPTL_OK;
}

// ------------------------------------------------------------- LayerNorm
bool ln_split(int h, int *tpr, int *vpt) {
  if (h <= 0 || h % 8) return false;
  const int v = h / 8;
  for (int limit : {5, 8})
    for (int t : {16, 32, 64, 128, 256})
      if (v % t == 0 && v / t >= 1 && v / t <= limit) {
        *tpr = t;
        *vpt = v / t;
        return true;
      }
  return false;
}

// Calls f.template operator()<VPT>() for the runtime vectors-per-thread.
template <typename F>
bool ln_dispatch(int vpt, F &&f) {
  switch (vpt) {
    case 1: f.template operator()<1>(); return true;
    case 2: f.template operator()<2>(); return true;
    case 3: f.template operator()<3>(); return true;
    case 4: f.template operator()<4>(); return true;
    case 5: f.template operator()<5>(); return true;
    case 6: f.template operator()<6>(); return true;
    case 7: f.template operator()<7>(); return true;
    case 8: f.template operator()<8>(); return true;
    default: return false;
  }
}

// Dynamic shared memory of ln_bwd_kernel with `nparts` running column sums
// per row team (0 when h has no split).  The kernel's static shared memory is
// under 1 KB; kLnBwdSmemMax keeps that margin below the opt-in limit.
constexpr int kLnBwdSmemMax = kSmemLimit - 1024;
long long ln_bwd_smem(int h, int nparts) {
  int tpr = 0, vpt = 0;
  if (!ln_split(h, &tpr, &vpt)) return 0;
  return (long long)(256 / tpr) * nparts * h * (long long)sizeof(float);
}

int ln_bwd_blocks(int rows, int h, int sms) {
  int tpr = 0, vpt = 0;
  if (!ln_split(h, &tpr, &vpt)) return 0;
  const int rpb = 256 / tpr;
  int nb = (rows + rpb - 1) / rpb;
  if (nb > 2 * sms) nb = 2 * sms;
  if (nb > 512) nb = 512;
  return nb;
}

// LayerNorm forward; x is 16-bit, or fp32 when x_f32.
int run_ln_fwd(int rows, int h, gptl_dtype dt, const void *x, int x_f32, const void *g,
               const void *b, float eps, void *y, float *mu, float *rstd, cudaStream_t st) {
  int tpr = 0, vpt = 0;
  if (!ln_split(h, &tpr, &vpt) || rows <= 0) return GPTL_E_SHAPE;
  const int rpb = 256 / tpr;
  const unsigned grid = (unsigned)((rows + rpb - 1) / rpb);
  const bool ok = ln_dispatch(vpt, [&]<int VP>() {
    auto go = [&]<typename T>() {
      if (x_f32)
        ln_fwd_kernel<T, float, VP><<<grid, 256, 0, st>>>((const float *)x, (const T *)g,
                                                          (const T *)b, (T *)y, mu, rstd, rows,
                                                          h, eps, tpr);
      else
        ln_fwd_kernel<T, T, VP><<<grid, 256, 0, st>>>((const T *)x, (const T *)g, (const T *)b,
                                                      (T *)y, mu, rstd, rows, h, eps, tpr);
    };
    if (dt == GPTL_FP16) go.template operator()<__half>();
    else go.template operator()<__nv_bfloat16>();
  });
  if (!ok) return GPTL_E_SHAPE;
  GPTL_CK(cudaGetLastError());
  prof_launched(st, GPTL_KIND_LN_FWD);
  return GPTL_OK;
}

int launch_reduce_parts(const float *part, int nblocks, int n, int nk, float *o0, float *o1,
                        float *o2, float *o3, cudaStream_t st) {
  PartOuts outs{{o0, o1, o2, o3}, g_nonfinite};
  reduce_parts_kernel<<<dim3((n + 31) / 32, nk), dim3(32, 16), 0, st>>>(part, nblocks, n, outs);
  GPTL_CK(cudaGetLastError());
  prof_launched(st, GPTL_KIND_REDUCE);
  return GPTL_OK;
}

// LayerNorm backward in the three arrangements the library uses:
//   LNB_PARTS : x, resid 16-bit; dx 16-bit; sums dg, db [, dx];
//   LNB_H     : x fp32 (the residual stream H), resid 16-bit (dOut); dx written
//               16-bit and fp32; sums dg, db, dx (fp32 value), resid;
//   LNB_X     : x 16-bit (the layer input), resid fp32 (dH); dx 16-bit; sums dg, db.
enum { LNB_PARTS = 0, LNB_H = 1, LNB_X = 2 };

int run_ln_bwd(int variant, int rows, int h, gptl_dtype dt, const void *gy, const void *x,
               const float *mu, const float *rstd, const void *g, const void *resid, void *dx,
               float *dx32, float *dg, float *db, float *dx_sum, float *resid_sum, float *part,
               cudaStream_t st) {
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  int tpr = 0, vpt = 0;
  if (!ln_split(h, &tpr, &vpt) || rows <= 0) return GPTL_E_SHAPE;
  const int nb = ln_bwd_blocks(rows, h, sms);
  const int nparts = variant == LNB_H ? 4 : (variant == LNB_X ? 2 : (dx_sum ? 3 : 2));
  const long long smem_ll = ln_bwd_smem(h, nparts);   // per-team running sums
  if (smem_ll <= 0 || smem_ll > kLnBwdSmemMax) return GPTL_E_SHAPE;
  const int smem = (int)smem_ll;
  int rc = GPTL_OK;
  const bool ok = ln_dispatch(vpt, [&]<int VP>() {
    auto go = [&]<typename T, typename TX, typename TR, bool D32, bool SDX, bool SRS>() {
      auto kern = ln_bwd_kernel<T, TX, TR, D32, SDX, SRS, VP>;
      if (smem > 40 * 1024 &&   // the opt-in also covers the kernel's static shared memory
          cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
              cudaSuccess) {
        (void)cudaGetLastError();
        rc = GPTL_E_CUDA;
        return;
      }
      kern<<<nb, 256, smem, st>>>((const T *)gy, (const TX *)x, mu, rstd, (const T *)g,
                                  (const TR *)resid, (T *)dx, dx32, part, rows, h, tpr);
    };
    auto by_variant = [&]<typename T>() {
      if (variant == LNB_H) go.template operator()<T, float, T, true, true, true>();
      else if (variant == LNB_X) go.template operator()<T, T, float, false, false, false>();
      else if (dx_sum) go.template operator()<T, T, T, false, true, false>();
      else go.template operator()<T, T, T, false, false, false>();
    };
    if (dt == GPTL_FP16) by_variant.template operator()<__half>();
    else by_variant.template operator()<__nv_bfloat16>();
  });
  if (!ok) return GPTL_E_SHAPE;
  GPTL_TRY(rc);
  GPTL_CK(cudaGetLastError());
  prof_launched(st, GPTL_KIND_LN_BWD);
  if (variant == LNB_H) return launch_reduce_parts(part, nb, h, 4, dg, db, dx_sum, resid_sum, st);
  if (variant == LNB_X) return launch_reduce_parts(part, nb, h, 2, dg, db, nullptr, nullptr, st);
  return launch_reduce_parts(part, nb, h, dx_sum ? 3 : 2, dg, db, dx_sum, nullptr, st);
}

// ------------------------------------------------------------- col sums
constexpr int kColsumMaxSplit = 64;

int run_colsum(int rows, int n, int groups, long long ld, long long gstride, gptl_dtype dt,
               const void *a, float *out, float *part, cudaStream_t st) {
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  if (rows <= 0 || n <= 0 || groups <= 0 || n % 8 || ld % 8 || (groups > 1 && gstride % 8))
    return GPTL_E_SHAPE;
  const int strips = (n + 255) / 256;
  // enough blocks for ~8 per SM (bytes in flight for HBM bandwidth)
  int split = (8 * sms + strips * groups - 1) / (strips * groups);
  if (split < 1) split = 1;
  if (split > kColsumMaxSplit) split = kColsumMaxSplit;
  if (split > (rows + 7) / 8) split = (rows + 7) / 8;
  dim3 grid(strips, split, groups), block(32, 8);
  if (dt == GPTL_FP16)
    colsum_kernel<__half><<<grid, block, 0, st>>>((const __half *)a, rows, n, ld, gstride, part,
                                                  groups);
  else
    colsum_kernel<__nv_bfloat16><<<grid, block, 0, st>>>((const __nv_bfloat16 *)a, rows, n, ld,
                                                         gstride, part, groups);
  GPTL_CK(cudaGetLastError());
  prof_launched(st, GPTL_KIND_COLSUM);
  const int width = n * groups;
  return launch_reduce_parts(part, split, width, 1, out, nullptr, nullptr, nullptr, st);
}

// Fixed partial-sum storage of gptl_colsum_noalloc: kColsumMaxSplit partial
// rows of at most kNoAllocMaxWidth columns.  Host code may not use the
// array's name as a device address; noalloc_scratch() looks the address up
// with the device current, once per CUDA context: the cached address is kept
// with the id of the context it came from, so that a device reset (which
// ends the context and the array's old mapping with it) leads to a fresh
// lookup instead of a stale pointer.  A mutex guards the table, which host
// threads share.
constexpr int kNoAllocMaxWidth = 16384;
static __device__ __align__(256) float g_colsum_scratch[(size_t)kColsumMaxSplit * kNoAllocMaxWidth];
struct NoAllocSlot {
  unsigned long long ctx_id;
  float *addr;
};
NoAllocSlot g_colsum_scratch_slot[kMaxDevices];
std::mutex g_colsum_scratch_mu;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

// Id of the calling thread's current CUDA context, or 0 when there is none
// (or the driver cannot say).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(p);
    (void)cudaGetLastError();
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

int noalloc_scratch(float **out) {
  int dev = 0;
  GPTL_CK(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return GPTL_E_ARCH;
  GPTL_TRY(device_check());
  std::lock_guard<std::mutex> lock(g_colsum_scratch_mu);
  NoAllocSlot &slot = g_colsum_scratch_slot[dev];
  const unsigned long long id = current_context_id();
  if (!slot.addr || id == 0 || slot.ctx_id != id) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_colsum_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return GPTL_E_CUDA;
    }
    slot.addr = static_cast<float *>(p);
    slot.ctx_id = current_context_id();   // the lookup made the context current if it was not
  }
  *out = slot.addr;
  return GPTL_OK;
}

// ------------------------------------------------------------- the layer
struct Dims {
  int b, s, h, a, f, t, d, hs, as, fs;
  long long T;
  gptl_dtype dt;
  float eps;
  int recompute;   // the FFN activation A is recomputed in the backward, not saved
};

int check_shape(const gptl_shape *sh, Dims *D) {
  if (!sh) return GPTL_E_NULL;
  if (sh->dtype != GPTL_FP16 && sh->dtype != GPTL_BF16) return GPTL_E_DTYPE;
  const int b = sh->batch, s = sh->seq, h = sh->hidden, a = sh->heads, f = sh->ffn, t = sh->tp;
  if (b <= 0 || s <= 0 || h <= 0 || a <= 0 || f <= 0 || t <= 0) return GPTL_E_SHAPE;
  if (h % a || a % t || f % t) return GPTL_E_SHAPE;
  const int d = h / a;
  if (d % 16 || d > 128 || h % 64 || (f / t) % 64 || s % 16 || s > 2048) return GPTL_E_SHAPE;
  if ((long long)b * s >= (1ll << 31)) return GPTL_E_SHAPE;
  if (!(sh->ln_eps > 0.f)) return GPTL_E_SHAPE;
  if (sh->recompute_gelu != 0 && sh->recompute_gelu != 1) return GPTL_E_SHAPE;
  int tpr, vpt;
  if (!ln_split(h, &tpr, &vpt)) return GPTL_E_SHAPE;
  // every launch-time limit of the step is checked here, so that no call
  // fails after its first launch: the LayerNorm backward's running sums (four
  // per row team in the LayerNorm-2 backward) must fit in shared memory.  The
  // attention kernels' shared memory fits for every d <= 128, and the GEMM's
  // stages for every tile it picks.
  if (ln_bwd_smem(h, 4) > kLnBwdSmemMax) return GPTL_E_SHAPE;
  D->b = b; D->s = s; D->h = h; D->a = a; D->f = f; D->t = t; D->d = d;
  D->hs = h / t; D->as = a / t; D->fs = f / t;
  D->T = (long long)b * s;
  D->dt = sh->dtype;
  D->eps = sh->ln_eps;
  D->recompute = sh->recompute_gelu;
  return GPTL_OK;
}

struct Ws {
  // saved (fwd -> bwd)
  size_t mu1, rstd1, mu2, rstd2, l1, c, lse, o, hid, l2, z, act, saved;
  // scratch (bwd)
  size_t dz, dl2, dhid, dhid32, dO, dvec, dc, dl1, xt, w2t, w1t, wot, wqkvt, part, splitk,
      splitk_bytes, scratch;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

Ws ws_layout(const Dims &D) {
  Ws w;
  const size_t e = 2, T = (size_t)D.T, h = D.h, f = D.f;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += up256(bytes);
    return o;
  };
  w.mu1 = take(T * 4); w.rstd1 = take(T * 4); w.mu2 = take(T * 4); w.rstd2 = take(T * 4);
  w.l1 = take(T * h * e); w.c = take(3 * T * h * e);
  w.lse = take((size_t)D.b * D.a * D.s * 4);   // attention row log-sum-exp, fp32
  w.o = take(T * h * e);
  w.hid = take(T * h * 4);             // residual stream H, fp32
  w.l2 = take(T * h * e); w.z = take(T * f * e);
  if (!D.recompute) w.act = take(T * f * e);
  w.saved = off;
  off = 0;
  // with recompute, A = GeLU(Z) lives in scratch: the forward writes it for
  // FFN2, the backward writes it again from the saved Z
  if (D.recompute) w.act = take(T * f * e);
  w.dz = take(T * f * e); w.dl2 = take(T * h * e); w.dhid = take(T * h * e);
  w.dhid32 = take(T * h * 4);          // residual-stream gradient dH, fp32
  w.dO = take(T * h * e);
  w.dvec = take((size_t)D.b * D.a * D.s * 4);
  w.dc = take(3 * T * h * e); w.dl1 = take(T * h * e);
  w.xt = take(T * h * e);               // [h][T] transposed operand of a weight gradient
  // transposed 16-bit weights ([in][out] per shard) for the input-gradient GEMMs
  w.w2t = take(h * f * e); w.w1t = take(f * h * e); w.wot = take(h * h * e);
  w.wqkvt = take(3 * h * h * e);
  // partial sums: the LayerNorm backward's, the column-sum pass's (db_1) and
  // the 32-row column sums of dC (b * ceil(s/32) rows of 3h)
  size_t part = 4 * 512 * h;
  const size_t widest = f > 3 * h ? f : 3 * h;
  if (kColsumMaxSplit * widest > part) part = kColsumMaxSplit * widest;
  const size_t cs_rows = (size_t)D.b * ((D.s + 31) / 32);
  if (cs_rows * 3 * h > part) part = cs_rows * 3 * h;
  w.part = take(part * 4);
  // split-K partials of the weight-gradient GEMMs: up to 8 slices of the
  // largest gradient, at most 64 MiB (large layers have tiles enough)
  size_t sk = (size_t)8 * h * (f > 3 * h ? f : 3 * h) * 4;
  if (sk > ((size_t)64 << 20)) sk = (size_t)64 << 20;
  w.splitk_bytes = sk;
  w.splitk = take(sk);
  w.scratch = off;
  return w;
}

template <typename P> P *at(void *base, size_t off) {
  return reinterpret_cast<P *>(static_cast<char *>(base) + off);
}
template <typename P> const P *at(const void *base, size_t off) {
  return reinterpret_cast<const P *>(static_cast<const char *>(base) + off);
}

constexpr int kNoGroup = 1 << 30;

gptl_operand view(const void *ptr, long long x_ext, long long rows, long long g_ext,
                  long long row_pitch, long long g_pitch, int mn) {
  gptl_operand o;
  o.ptr = ptr;
  o.x_ext = x_ext;
  o.rows_ext = rows;
  o.g_ext = g_ext;
  o.row_pitch = row_pitch;
  o.g_pitch = g_pitch;
  o.mn_major = mn;
  o.x_mod = 1;
  o.x_mul = 0;
  o.x_off = 0;
  o.g_div = g_ext > 1 ? 1 : kNoGroup;
  o.k_shard = 0;
  return o;
}

gptl_gemm_desc gemm(int M, int N, int K, int groups, const gptl_operand &a, const gptl_operand &b,
                    void *out, long long ldo, long long o_str_div) {
  gptl_gemm_desc d;
  memset(&d, 0, sizeof(d));
  d.M = M; d.N = N; d.K = K; d.groups = groups; d.k_shards = 1;
  d.a = a; d.b = b;
  d.out = out; d.ldo = ldo; d.o_mod = 1; d.o_str_div = o_str_div;
  return d;
}

int validate_weights(const gptl_weights *w) {
  if (!w) return GPTL_E_NULL;
  const void *ps[12] = {w->ln1_g, w->ln1_b, w->w_qkv, w->b_qkv, w->w_o, w->b_o,
                        w->ln2_g, w->ln2_b, w->w_1, w->b_1, w->w_2, w->b_2};
  for (const void *p : ps) {
    if (!p) return GPTL_E_NULL;
    if (!aligned16(p)) return GPTL_E_ALIGN;
  }
  // the transposed copies: all four or none
  const void *ts[4] = {w->w_qkv_t, w->w_o_t, w->w_1_t, w->w_2_t};
  int given = 0;
  for (const void *p : ts) {
    if (!p) continue;
    ++given;
    if (!aligned16(p)) return GPTL_E_ALIGN;
  }
  if (given != 0 && given != 4) return GPTL_E_NULL;
  return GPTL_OK;
}

// The four weight matrices transposed shard by shard (one launch): the
// layout gptl_weights' *_t fields describe.
int run_weight_transposes(const Dims &D, const gptl_weights *W, void *wqkvt, void *wot, void *w1t,
                          void *w2t, cudaStream_t st) {
  const int h = D.h, t = D.t, hs = D.hs, fs = D.fs;
  const TransposeSpec wt[4] = {
      {h, fs, W->w_2, fs, w2t, h, t, (long long)h * fs, (long long)fs * h},
      {fs, h, W->w_1, h, w1t, fs, t, (long long)fs * h, (long long)h * fs},
      {h, hs, W->w_o, hs, wot, h, t, (long long)h * hs, (long long)hs * h},
      {3 * hs, h, W->w_qkv, h, wqkvt, 3 * hs, t, (long long)3 * hs * h, (long long)h * 3 * hs}};
  return run_transposes(wt, 4, st);
}

int layer_fwd(const Dims &D, const gptl_weights *W, const void *x, void *y, void *saved,
              void *scratch, cudaStream_t st) {
  const Ws w = ws_layout(D);
  const gptl_dtype dt = D.dt;
  const int T = (int)D.T, h = D.h, t = D.t, s = D.s, d = D.d, hs = D.hs, as = D.as, fs = D.fs;
  void *l1 = at<void>(saved, w.l1), *c = at<void>(saved, w.c);
  float *lse = at<float>(saved, w.lse);
  void *o = at<void>(saved, w.o), *hid = at<void>(saved, w.hid), *l2 = at<void>(saved, w.l2);
  void *z = at<void>(saved, w.z);
  void *act = D.recompute ? at<void>(scratch, w.act) : at<void>(saved, w.act);
  float *mu1 = at<float>(saved, w.mu1), *rs1 = at<float>(saved, w.rstd1);
  float *mu2 = at<float>(saved, w.mu2), *rs2 = at<float>(saved, w.rstd2);
  TagScope tag_scope(GPTL_TAG_NONE);
  prof_start(st);

  // LN1
  g_tag = GPTL_TAG_F1_LN1;
  GPTL_TRY(run_ln_fwd(T, h, dt, x, 0, W->ln1_g, W->ln1_b, D.eps, l1, mu1, rs1, st));
  // QKV column split: C_i = L1 W_qkv,i^T + b_qkv,i
  g_tag = GPTL_TAG_F2_QKV;
  {
    gptl_gemm_desc g = gemm(T, 3 * hs, h, t, view(l1, h, T, 1, h, 0, 0),
                            view(W->w_qkv, h, 3 * hs, t, h, (long long)3 * hs * h, 0), c, 3 * hs,
                            (long long)T * 3 * hs);
    g.bias = W->b_qkv;
    g.bias_g_stride = 3 * hs;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  // causal attention, fused: S, softmax and P stay on chip; O and the
  // row log-sum-exp go to memory
  g_tag = GPTL_TAG_F3_F5_ATTN;
  GPTL_TRY(run_attn_fwd(D.b, s, hs, as, t, d, dt, c, o, lse, st));
  // out-projection, row split: H = X + sum_i O_i W_o,i^T + b_o
  g_tag = GPTL_TAG_F6_OUTPROJ;
  {
    gptl_operand a = view(o, hs, T, t, hs, (long long)T * hs, 0);
    a.g_div = kNoGroup; a.k_shard = 1;
    gptl_operand b = view(W->w_o, hs, h, t, hs, (long long)h * hs, 0);
    b.g_div = kNoGroup; b.k_shard = 1;
    gptl_gemm_desc g = gemm(T, h, hs, 1, a, b, hid, h, 0);
    g.k_shards = t;
    g.out_f32 = 1;                       // H stays fp32 (the residual stream)
    g.bias = W->b_o;
    g.resid = x;
    g.ld_resid = h;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  // LN2
  g_tag = GPTL_TAG_F7_LN2;
  GPTL_TRY(run_ln_fwd(T, h, dt, hid, 1, W->ln2_g, W->ln2_b, D.eps, l2, mu2, rs2, st));
  // FFN1 column split with fused bias + GeLU: Z_i, A_i = gelu(Z_i)
  g_tag = GPTL_TAG_F8_FFN1_GELU;
  {
    gptl_gemm_desc g = gemm(T, fs, h, t, view(l2, h, T, 1, h, 0, 0),
                            view(W->w_1, h, fs, t, h, (long long)fs * h, 0), z, fs,
                            (long long)T * fs);
    g.bias = W->b_1;
    g.bias_g_stride = fs;
    g.act = GPTL_ACT_GELU;
    g.out2 = act;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  // FFN2 row split: Out = H + sum_i A_i W_2,i^T + b_2
  g_tag = GPTL_TAG_F10_FFN2;
  {
    gptl_operand a = view(act, fs, T, t, fs, (long long)T * fs, 0);
    a.g_div = kNoGroup; a.k_shard = 1;
    gptl_operand b = view(W->w_2, fs, h, t, fs, (long long)h * fs, 0);
    b.g_div = kNoGroup; b.k_shard = 1;
    gptl_gemm_desc g = gemm(T, h, fs, 1, a, b, y, h, 0);
    g.k_shards = t;
    g.bias = W->b_2;
    g.resid = hid;
    g.resid_f32 = 1;
    g.ld_resid = h;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  return GPTL_OK;
}

int layer_bwd(const Dims &D, const gptl_weights *W, const void *x, const void *saved,
              const void *dy, void *dx, const gptl_grads *gr, void *scratch, cudaStream_t st) {
  const Ws w = ws_layout(D);
  const gptl_dtype dt = D.dt;
  const int T = (int)D.T, h = D.h, t = D.t, s = D.s, d = D.d, hs = D.hs, as = D.as, fs = D.fs;
  const void *l1 = at<void>(saved, w.l1), *c = at<void>(saved, w.c);
  const float *lse = at<float>(saved, w.lse);
  const void *o = at<void>(saved, w.o), *hid = at<void>(saved, w.hid);
  const void *l2 = at<void>(saved, w.l2), *z = at<void>(saved, w.z);
  // A = GeLU(Z): saved by the forward, or (recompute) written again below
  void *act_re = D.recompute ? at<void>(scratch, w.act) : nullptr;
  const void *act = D.recompute ? act_re : at<void>(saved, w.act);
  const float *mu1 = at<float>(saved, w.mu1), *rs1 = at<float>(saved, w.rstd1);
  const float *mu2 = at<float>(saved, w.mu2), *rs2 = at<float>(saved, w.rstd2);
  void *dz = at<void>(scratch, w.dz), *dl2 = at<void>(scratch, w.dl2);
  float *dhid32 = at<float>(scratch, w.dhid32);
  void *dhid = at<void>(scratch, w.dhid), *dO = at<void>(scratch, w.dO);
  void *dc = at<void>(scratch, w.dc), *dl1 = at<void>(scratch, w.dl1);
  float *dvec = at<float>(scratch, w.dvec);
  void *xt = at<void>(scratch, w.xt);   // [h][T]: one token-contiguous copy at a time
  // the transposed weights: the caller's copies, or transposed below
  const bool own_wt = W->w_qkv_t == nullptr;
  const void *w2t = own_wt ? at<void>(scratch, w.w2t) : W->w_2_t;
  const void *w1t = own_wt ? at<void>(scratch, w.w1t) : W->w_1_t;
  const void *wot = own_wt ? at<void>(scratch, w.wot) : W->w_o_t;
  const void *wqkvt = own_wt ? at<void>(scratch, w.wqkvt) : W->w_qkv_t;
  float *part = at<float>(scratch, w.part);
  void *splitk = at<void>(scratch, w.splitk);
  const long long splitk_bytes = (long long)w.splitk_bytes;
  const float attn_scale = 1.0f / sqrtf((float)d);
  TagScope tag_scope(GPTL_TAG_NONE);
  prof_start(st);

  // The input-gradient GEMMs read the weights with the reduction index
  // contiguous: transposed copies, shard by shard (unless the caller's
  // optimizer step wrote them already).
  g_tag = GPTL_TAG_B0_WT;
  if (own_wt) GPTL_TRY(run_weight_transposes(D, W, at<void>(scratch, w.wqkvt), at<void>(scratch, w.wot),
                                             at<void>(scratch, w.w1t), at<void>(scratch, w.w2t), st));

  // ---- FFN2 (row split)
  // Weight gradients reduce over the tokens, the row index of both
  // activations; the tensor core runs markedly faster when one operand is
  // token-contiguous, so the smaller operand is transposed first.
  g_tag = GPTL_TAG_B2_DOUT_T;
  GPTL_TRY(run_transpose(T, h, dy, h, xt, T, st));
  g_tag = GPTL_TAG_B1_B3_DZ;
  {  // dZ_i = (dOut W2_i) * gelu'(Z_i)
    // (db_1 is a separate column-sum pass below: summing in this GEMM's
    // epilogue, which its tensor-memory load latency already bounds, measured
    // slower at both the GPT-2 117M and the hidden-10240 shapes)
    gptl_gemm_desc g = gemm(T, fs, h, t, view(dy, h, T, 1, h, 0, 0),
                            view(w2t, h, fs, t, h, (long long)fs * h, 0), dz, fs,
                            (long long)T * fs);
    g.act = GPTL_ACT_DGELU;
    g.aux = z;
    g.out2 = act_re;                     // recompute: A_i = gelu(Z_i) again, for dW2
    GPTL_TRY(run_gemm(g, dt, st));
  }
  g_tag = GPTL_TAG_B2_DW2;
  {  // dW2_i = dOut^T A_i   [t][h][f/t] fp32
    gptl_gemm_desc g = gemm(h, fs, T, t, view(xt, T, h, 1, T, 0, 0),
                            view(act, fs, T, t, fs, (long long)T * fs, 1), gr->w_2, fs,
                            (long long)h * fs);
    g.out_f32 = 1;
    g.ws = splitk;
    g.ws_bytes = splitk_bytes;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  // ---- FFN1 (column split)
  g_tag = GPTL_TAG_B3_DB1;
  GPTL_TRY(run_colsum(T, fs, t, fs, (long long)T * fs, dt, dz, gr->b_1, part, st));
  g_tag = GPTL_TAG_B5_L2_T;
  GPTL_TRY(run_transpose(T, h, l2, h, xt, T, st));
  g_tag = GPTL_TAG_B5_DW1;
  {  // dW1_i = dZ_i^T L2   [t][f/t][h]
    gptl_gemm_desc g = gemm(fs, h, T, t, view(dz, fs, T, t, fs, (long long)T * fs, 1),
                            view(xt, T, h, 1, T, 0, 0), gr->w_1, h, (long long)fs * h);
    g.out_f32 = 1;
    g.ws = splitk;
    g.ws_bytes = splitk_bytes;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  g_tag = GPTL_TAG_B4_DL2;
  {  // dL2 = sum_i dZ_i W1_i  (shard sum in the K loop)
    gptl_operand a = view(dz, fs, T, t, fs, (long long)T * fs, 0);
    a.g_div = kNoGroup; a.k_shard = 1;
    gptl_operand b = view(w1t, fs, h, t, fs, (long long)h * fs, 0);
    b.g_div = kNoGroup; b.k_shard = 1;
    gptl_gemm_desc g = gemm(T, h, fs, 1, a, b, dl2, h, 0);
    g.k_shards = t;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  // ---- LN2 backward + residual: dH = dOut + LNbwd(dL2); also db_o = sum dH
  g_tag = GPTL_TAG_B6_LN2;
  //      (the same pass sums dH into db_o and dOut into db_2)
  GPTL_TRY(run_ln_bwd(LNB_H, T, h, dt, dl2, hid, mu2, rs2, W->ln2_g, dy, dhid, dhid32, gr->ln2_g,
                      gr->ln2_b, gr->b_o, gr->b_2, part, st));
  // ---- out-projection (row split)
  g_tag = GPTL_TAG_B7_DH_T;
  GPTL_TRY(run_transpose(T, h, dhid, h, xt, T, st));
  g_tag = GPTL_TAG_B7_DWO;
  {  // dWo_i = dH^T O_i   [t][h][h/t]
    gptl_gemm_desc g = gemm(h, hs, T, t, view(xt, T, h, 1, T, 0, 0),
                            view(o, hs, T, t, hs, (long long)T * hs, 1), gr->w_o, hs,
                            (long long)h * hs);
    g.out_f32 = 1;
    g.ws = splitk;
    g.ws_bytes = splitk_bytes;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  g_tag = GPTL_TAG_B7_DO;
  {  // dO_i = dH Wo_i   [t][T][h/t]
    gptl_gemm_desc g = gemm(T, hs, h, t, view(dhid, h, T, 1, h, 0, 0),
                            view(wot, h, hs, t, h, (long long)hs * h, 0), dO, hs,
                            (long long)T * hs);
    GPTL_TRY(run_gemm(g, dt, st));
  }
  // ---- attention backward
  g_tag = GPTL_TAG_B9_ROWDOT;   // D = rowsum(dO * O), the softmax backward's row term
  GPTL_TRY(run_attn_rowdot((long long)t * T, s, hs, as, d, dt, dO, o, dvec, st));
  // fused attention backward: dQ, dK, dV into dC (P and dS stay on chip),
  // with the 32-row column sums of dC (db_qkv's partials)
  g_tag = GPTL_TAG_B8_B10_ATTN;
  GPTL_TRY(run_attn_bwd(D.b, s, hs, as, t, d, dt, c, dO, lse, dvec, dc, part, st));
  // ---- QKV (column split)
  g_tag = GPTL_TAG_B11_DBQKV;
  GPTL_TRY(launch_reduce_parts(part, D.b * ((s + 31) / 32), t * 3 * hs, 1, gr->b_qkv, nullptr,
                               nullptr, nullptr, st));
  g_tag = GPTL_TAG_B11_L1_T;
  GPTL_TRY(run_transpose(T, h, l1, h, xt, T, st));
  g_tag = GPTL_TAG_B11_DWQKV;
  {  // dWqkv_i = dC_i^T L1   [t][3h/t][h]
    gptl_gemm_desc g = gemm(3 * hs, h, T, t, view(dc, 3 * hs, T, t, 3 * hs, (long long)T * 3 * hs, 1),
                            view(xt, T, h, 1, T, 0, 0), gr->w_qkv, h, (long long)3 * hs * h);
    g.out_f32 = 1;
    g.ws = splitk;
    g.ws_bytes = splitk_bytes;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  g_tag = GPTL_TAG_B11_DL1;
  {  // dL1 = sum_i dC_i Wqkv_i
    gptl_operand a = view(dc, 3 * hs, T, t, 3 * hs, (long long)T * 3 * hs, 0);
    a.g_div = kNoGroup; a.k_shard = 1;
    gptl_operand b = view(wqkvt, 3 * hs, h, t, 3 * hs, (long long)h * 3 * hs, 0);
    b.g_div = kNoGroup; b.k_shard = 1;
    gptl_gemm_desc g = gemm(T, h, 3 * hs, 1, a, b, dl1, h, 0);
    g.k_shards = t;
    GPTL_TRY(run_gemm(g, dt, st));
  }
  // ---- LN1 backward + residual: dX = dH + LNbwd(dL1)
  g_tag = GPTL_TAG_B12_LN1;
  GPTL_TRY(run_ln_bwd(LNB_X, T, h, dt, dl1, x, mu1, rs1, W->ln1_g, dhid32, dx, nullptr,
                      gr->ln1_g, gr->ln1_b, nullptr, nullptr, part, st));
  return GPTL_OK;
}

}  // namespace

// =================================================================== C ABI
extern "C" {

const char *gptl_strerror(int code) {
  switch (code) {
    case GPTL_OK: return "ok";
    case GPTL_E_NULL: return "a required pointer is NULL";
    case GPTL_E_SHAPE: return "unsupported or inconsistent sizes";
    case GPTL_E_ALIGN: return "a pointer or pitch is not 16-byte aligned";
    case GPTL_E_DTYPE: return "dtype must be GPTL_FP16 or GPTL_BF16";
    case GPTL_E_ARCH: return "the current device is not compute capability 10.x (sm_100a)";
    case GPTL_E_CUDA: return "a CUDA call or kernel launch failed";
    case GPTL_E_DEVICE: return "the device error word is set";
    case GPTL_E_ARG: return "invalid scalar argument";
    case GPTL_E_TOO_LARGE: return "the sizes exceed a fixed internal capacity";
    default: return "unknown error";
  }
}

int gptl_read_device_error(int *word, int clear) {
  if (!word) return GPTL_E_NULL;
  GPTL_CK(cudaDeviceSynchronize());
  GPTL_CK(cudaMemcpyFromSymbol(word, g_device_error, sizeof(int)));
  if (clear) {
    const int zero = 0;
    GPTL_CK(cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)));
  }
  return GPTL_OK;
}

int gpt_layer_workspace_bytes(const gptl_shape *shape, size_t *saved_bytes, size_t *scratch_bytes) {
  Dims D;
  GPTL_TRY(check_shape(shape, &D));
  if (!saved_bytes || !scratch_bytes) return GPTL_E_NULL;
  const Ws w = ws_layout(D);
  *saved_bytes = w.saved;
  *scratch_bytes = w.scratch;
  return GPTL_OK;
}

int gpt_layer_param_layout(const gptl_shape *shape, size_t offsets[12], size_t *n_params) {
  Dims D;
  GPTL_TRY(check_shape(shape, &D));
  if (!offsets || !n_params) return GPTL_E_NULL;
  const size_t h = D.h, f = D.f;
  const size_t sizes[12] = {h, h, 3 * h * h, 3 * h, h * h, h, h, h, f * h, f, h * f, h};
  size_t off = 0;
  for (int i = 0; i < 12; ++i) {
    offsets[i] = off;
    off += (sizes[i] + 63) / 64 * 64;
  }
  *n_params = off;
  return GPTL_OK;
}

int gpt_layer_fwd(const gptl_shape *shape, const gptl_weights *w, const void *x, void *y,
                  void *saved, void *scratch, gptl_stream_t stream) {
  Dims D;
  GPTL_TRY(check_shape(shape, &D));
  GPTL_TRY(validate_weights(w));
  if (!x || !y || !saved || (D.recompute && !scratch)) return GPTL_E_NULL;
  if (!aligned16(x) || !aligned16(y) || !aligned16(saved) || (scratch && !aligned16(scratch)))
    return GPTL_E_ALIGN;
  GPTL_TRY(device_check());
  return layer_fwd(D, w, x, y, saved, scratch, reinterpret_cast<cudaStream_t>(stream));
}

namespace {
int bwd_validate(const gptl_shape *shape, const gptl_weights *w, const void *x, const void *saved,
                 const void *dy, void *dx, const gptl_grads *g, void *scratch, Dims *D) {
  GPTL_TRY(check_shape(shape, D));
  GPTL_TRY(validate_weights(w));
  if (!x || !saved || !dy || !dx || !g || !scratch) return GPTL_E_NULL;
  if (!aligned16(x) || !aligned16(saved) || !aligned16(dy) || !aligned16(dx) || !aligned16(scratch))
    return GPTL_E_ALIGN;
  const float *gp[12] = {g->ln1_g, g->ln1_b, g->w_qkv, g->b_qkv, g->w_o, g->b_o,
                         g->ln2_g, g->ln2_b, g->w_1, g->b_1, g->w_2, g->b_2};
  for (const float *p : gp) {
    if (!p) return GPTL_E_NULL;
    if (!aligned16(p)) return GPTL_E_ALIGN;
  }
  return device_check();
}

int adam_validate(size_t n_params, float *master, float *m, float *v, const float *grad, void *w16,
                  gptl_dtype dtype, float lr, float beta1, float beta2, float eps,
                  float weight_decay, gptl_scaler_state *st) {
  if (!master || !m || !v || !grad || !w16 || !st) return GPTL_E_NULL;
  if (dtype != GPTL_FP16 && dtype != GPTL_BF16) return GPTL_E_DTYPE;
  if (!aligned16(master) || !aligned16(m) || !aligned16(v) || !aligned16(grad) || !aligned16(w16) ||
      (reinterpret_cast<uintptr_t>(st) & 3u))
    return GPTL_E_ALIGN;
  if (n_params == 0 || n_params % 4 || !(lr >= 0.f) || !(beta1 >= 0.f && beta1 < 1.f) ||
      !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f) || !(weight_decay >= 0.f))
    return GPTL_E_ARG;
  return device_check();
}

// O2: the fused unscale + Adam + cast kernel; skips itself when st->found_inf.
int launch_adam(size_t n_params, float *master, float *m, float *v, const float *grad, void *w16,
                gptl_dtype dtype, float lr, float beta1, float beta2, float eps,
                float weight_decay, gptl_scaler_state *st, cudaStream_t s) {
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  const long long n4 = (long long)(n_params / 4);
  long long blocks = (n4 + 255) / 256;
  if (blocks > 8 * sms) blocks = 8 * sms;
  AdamArgs a{lr, beta1, beta2, eps, weight_decay};
  if (dtype == GPTL_FP16)
    adam_kernel<__half><<<(unsigned)blocks, 256, 0, s>>>(
        reinterpret_cast<float4 *>(master), reinterpret_cast<float4 *>(m),
        reinterpret_cast<float4 *>(v), reinterpret_cast<const float4 *>(grad),
        static_cast<__half *>(w16), n4, a, st);
  else
    adam_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
        reinterpret_cast<float4 *>(master), reinterpret_cast<float4 *>(m),
        reinterpret_cast<float4 *>(v), reinterpret_cast<const float4 *>(grad),
        static_cast<__nv_bfloat16 *>(w16), n4, a, st);
  GPTL_CK(cudaGetLastError());
  prof_launched(s, GPTL_KIND_ADAM);
  return GPTL_OK;
}

// Element offsets of the 12 parameter tensors in one layer's arena (the
// layout gpt_layer_param_layout reports) and its length.
void param_offsets(const Dims &D, size_t off[12], size_t *n_params) {
  const size_t h = D.h, f = D.f;
  const size_t sizes[12] = {h, h, 3 * h * h, 3 * h, h * h, h, h, h, f * h, f, h * f, h};
  size_t o = 0;
  for (int i = 0; i < 12; ++i) {
    off[i] = o;
    o += (sizes[i] + 63) / 64 * 64;
  }
  *n_params = o;
}

// The optimizer step that also writes the transposed weight matrices
// (adam_wt_kernel): the plan lists each layer's four matrices (shards of
// [rows][cols]) and the five vector ranges between them.
int launch_adam_wt(const Dims &D, int n_layers, float *master, float *m, float *v,
                   const float *grad, void *w16, void *w16t, float lr, float beta1, float beta2,
                   float eps, float weight_decay, gptl_scaler_state *st, cudaStream_t s) {
  size_t off[12], n_params = 0;
  param_offsets(D, off, &n_params);
  AdamWtPlan P;
  memset(&P, 0, sizeof(P));
  const int h = D.h, hs = D.hs, fs = D.fs;
  // (tensor index, shard rows, shard cols): w_qkv, w_o, w_1, w_2
  const int mats[4][3] = {{2, 3 * hs, h}, {4, h, hs}, {8, fs, h}, {10, h, fs}};
  long long tiles = 0;
  for (int k = 0; k < 4; ++k) {
    AdamMat &M = P.mat[k];
    M.off = (long long)off[mats[k][0]];
    M.rows = mats[k][1];
    M.cols = mats[k][2];
    M.tiles_r = (M.rows + 63) / 64;
    M.tiles_c = (M.cols + 63) / 64;
    M.tile0 = tiles;
    tiles += (long long)D.t * M.tiles_r * M.tiles_c;
  }
  P.nmat = 4;
  P.mat_tiles = tiles;
  // the vectors: [ln1_g, w_qkv), [b_qkv, w_o), [b_o, w_1), [b_1, w_2), [b_2, end)
  const size_t vr[5][2] = {{off[0], off[2]}, {off[3], off[4]}, {off[5], off[8]}, {off[9], off[10]},
                           {off[11], n_params}};
  long long chunks = 0;
  for (int k = 0; k < 5; ++k) {
    AdamVec &V = P.vec[k];
    V.off = (long long)vr[k][0];
    V.len = (long long)(vr[k][1] - vr[k][0]);
    V.chunk0 = chunks;
    chunks += (V.len + 1023) / 1024;
  }
  P.nvec = 5;
  P.vec_chunks = chunks;
  P.shards = D.t;
  P.layer_stride = (long long)n_params;
  P.mat_blocks = (long long)n_layers * P.mat_tiles;
  const long long blocks = P.mat_blocks + (long long)n_layers * P.vec_chunks;
  if (blocks >= (1ll << 31)) return GPTL_E_SHAPE;
  AdamArgs a{lr, beta1, beta2, eps, weight_decay};
  if (D.dt == GPTL_FP16)
    adam_wt_kernel<__half><<<(unsigned)blocks, 256, 0, s>>>(
        master, m, v, grad, static_cast<__half *>(w16), static_cast<__half *>(w16t), P, a, st);
  else
    adam_wt_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
        master, m, v, grad, static_cast<__nv_bfloat16 *>(w16), static_cast<__nv_bfloat16 *>(w16t),
        P, a, st);
  GPTL_CK(cudaGetLastError());
  prof_launched(s, GPTL_KIND_ADAM);
  return GPTL_OK;
}
}  // namespace

int gpt_layer_adam_step(const gptl_shape *shape, int n_layers, float *master, float *m, float *v,
                        const float *grad, void *w16, void *w16t, float lr, float beta1,
                        float beta2, float eps, float weight_decay, int prechecked,
                        gptl_scaler_state *st, gptl_stream_t stream) {
  Dims D;
  GPTL_TRY(check_shape(shape, &D));
  if (n_layers < 1 || (prechecked != 0 && prechecked != 1)) return GPTL_E_ARG;
  size_t off[12], n_params = 0;
  param_offsets(D, off, &n_params);
  if (!w16t) return GPTL_E_NULL;
  if (!aligned16(w16t)) return GPTL_E_ALIGN;
  const size_t n_all = n_params * (size_t)n_layers;
  GPTL_TRY(adam_validate(n_all, master, m, v, grad, w16, D.dt, lr, beta1, beta2, eps,
                         weight_decay, st));
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TagScope tag_scope(GPTL_TAG_O1_OVERFLOW);
  if (!prechecked) {
    GPTL_TRY(gptl_check_overflow(n_all, grad, st, stream));
  } else {
    prof_start(s);
  }
  g_tag = GPTL_TAG_O2_ADAM;
  return launch_adam_wt(D, n_layers, master, m, v, grad, w16, w16t, lr, beta1, beta2, eps,
                        weight_decay, st, s);
}

int gpt_layer_transpose_weights(const gptl_shape *shape, int n_layers, const void *w16, void *w16t,
                                gptl_stream_t stream) {
  Dims D;
  GPTL_TRY(check_shape(shape, &D));
  if (n_layers < 1) return GPTL_E_ARG;
  if (!w16 || !w16t) return GPTL_E_NULL;
  if (!aligned16(w16) || !aligned16(w16t)) return GPTL_E_ALIGN;
  GPTL_TRY(device_check());
  size_t off[12], n_params = 0;
  param_offsets(D, off, &n_params);
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TagScope tag_scope(GPTL_TAG_B0_WT);
  prof_start(s);
  for (int l = 0; l < n_layers; ++l) {
    const size_t base = (size_t)l * n_params * 2;   // bytes
    auto in = [&](int i) { return static_cast<const void *>(static_cast<const char *>(w16) + base + off[i] * 2); };
    auto out = [&](int i) { return static_cast<void *>(static_cast<char *>(w16t) + base + off[i] * 2); };
    gptl_weights W;
    memset(&W, 0, sizeof(W));
    W.w_qkv = in(2);
    W.w_o = in(4);
    W.w_1 = in(8);
    W.w_2 = in(10);
    GPTL_TRY(run_weight_transposes(D, &W, out(2), out(4), out(8), out(10), s));
  }
  return GPTL_OK;
}

int gpt_layer_bwd_checked(const gptl_shape *shape, const gptl_weights *w, const void *x,
                          const void *saved, const void *dy, void *dx, const gptl_grads *g,
                          void *scratch, gptl_scaler_state *st, gptl_stream_t stream) {
  Dims D;
  if (!st) return GPTL_E_NULL;
  if (reinterpret_cast<uintptr_t>(st) & 3u) return GPTL_E_ALIGN;
  GPTL_TRY(bwd_validate(shape, w, x, saved, dy, dx, g, scratch, &D));
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  GPTL_CK(cudaMemsetAsync(&st->found_inf, 0, sizeof(int), s));
  NonfiniteScope scope(&st->found_inf);
  return layer_bwd(D, w, x, saved, dy, dx, g, scratch, s);
}

int adam_step_fp32_master_prechecked(size_t n_params, float *master, float *m, float *v,
                                     const float *grad, void *w16, gptl_dtype dtype, float lr,
                                     float beta1, float beta2, float eps, float weight_decay,
                                     gptl_scaler_state *st, gptl_stream_t stream) {
  GPTL_TRY(adam_validate(n_params, master, m, v, grad, w16, dtype, lr, beta1, beta2, eps,
                         weight_decay, st));
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TagScope tag_scope(GPTL_TAG_O2_ADAM);
  prof_start(s);
  return launch_adam(n_params, master, m, v, grad, w16, dtype, lr, beta1, beta2, eps, weight_decay,
                     st, s);
}

int gpt_layer_bwd(const gptl_shape *shape, const gptl_weights *w, const void *x, const void *saved,
                  const void *dy, void *dx, const gptl_grads *g, void *scratch,
                  gptl_stream_t stream) {
  Dims D;
  GPTL_TRY(bwd_validate(shape, w, x, saved, dy, dx, g, scratch, &D));
  return layer_bwd(D, w, x, saved, dy, dx, g, scratch, reinterpret_cast<cudaStream_t>(stream));
}

int gptl_check_overflow(size_t n, const float *grad, gptl_scaler_state *st, gptl_stream_t stream) {
  int sms = 0;
  if (!grad || !st) return GPTL_E_NULL;
  if (!aligned16(grad) || (reinterpret_cast<uintptr_t>(st) & 3u)) return GPTL_E_ALIGN;
  if (n == 0 || n % 4) return GPTL_E_ARG;
  GPTL_TRY(device_check(&sms));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  GPTL_CK(cudaMemsetAsync(&st->found_inf, 0, sizeof(int), s));
  const long long n4 = (long long)(n / 4);
  long long blocks = (n4 + 255) / 256;
  if (blocks > 4 * sms) blocks = 4 * sms;
  prof_start(s);
  overflow_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4 *>(grad), n4,
                                                   &st->found_inf);
  GPTL_CK(cudaGetLastError());
  prof_launched(s, GPTL_KIND_OVERFLOW);
  return GPTL_OK;
}

int adam_step_fp32_master(size_t n_params, float *master, float *m, float *v, const float *grad,
                          void *w16, gptl_dtype dtype, float lr, float beta1, float beta2, float eps,
                          float weight_decay, gptl_scaler_state *st, gptl_stream_t stream) {
  GPTL_TRY(adam_validate(n_params, master, m, v, grad, w16, dtype, lr, beta1, beta2, eps,
                         weight_decay, st));
  TagScope tag_scope(GPTL_TAG_O1_OVERFLOW);
  GPTL_TRY(gptl_check_overflow(n_params, grad, st, stream));
  g_tag = GPTL_TAG_O2_ADAM;
  return launch_adam(n_params, master, m, v, grad, w16, dtype, lr, beta1, beta2, eps, weight_decay,
                     st, reinterpret_cast<cudaStream_t>(stream));
}

int loss_scale_update(gptl_scaler_state *st, int growth_interval, float growth_factor,
                      float backoff_factor, float min_scale, gptl_stream_t stream) {
  if (!st) return GPTL_E_NULL;
  if (growth_interval < 1 || !(growth_factor >= 1.f) || !(backoff_factor > 0.f && backoff_factor <= 1.f) ||
      !(min_scale > 0.f))
    return GPTL_E_ARG;
  GPTL_TRY(device_check());
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  TagScope tag_scope(GPTL_TAG_O3_SCALE);
  prof_start(s);
  scale_update_kernel<<<1, 32, 0, s>>>(st, growth_interval, growth_factor, backoff_factor,
                                       min_scale);
  GPTL_CK(cudaGetLastError());
  prof_launched(s, GPTL_KIND_SCALE);
  return GPTL_OK;
}

// ---------------------------------------------------------------- parts
int gptl_gemm(const gptl_gemm_desc *d, gptl_dtype dtype, gptl_stream_t stream) {
  if (!d) return GPTL_E_NULL;
  prof_start(reinterpret_cast<cudaStream_t>(stream));
  return run_gemm(*d, dtype, reinterpret_cast<cudaStream_t>(stream));
}

int gptl_gemm_plan(const gptl_gemm_desc *d, gptl_dtype dtype, int *bn, int *split, int *mode) {
  if (!d || !bn || !split || !mode) return GPTL_E_NULL;
  int sms = 0;
  GPTL_TRY(device_check(&sms));
  GPTL_TRY(gemm_validate(*d, dtype));
  const GemmTiling tl = gemm_plan(*d, sms);
  *bn = tl.bn;
  *split = tl.split;
  *mode = tl.m2 ? GPTL_GEMM_M256 : (tl.pipe_k ? GPTL_GEMM_K_HALVES : GPTL_GEMM_ALTERNATE);
  return GPTL_OK;
}

int gptl_layernorm_fwd(int rows, int h, gptl_dtype dtype, const void *x, const void *g,
                       const void *b, float eps, void *y, float *mu, float *rstd,
                       gptl_stream_t stream) {
  if (!x || !g || !b || !y || !mu || !rstd) return GPTL_E_NULL;
  if (dtype != GPTL_FP16 && dtype != GPTL_BF16) return GPTL_E_DTYPE;
  if (!aligned16(x) || !aligned16(g) || !aligned16(b) || !aligned16(y)) return GPTL_E_ALIGN;
  if (!(eps > 0.f)) return GPTL_E_ARG;
  GPTL_TRY(device_check());
  prof_start(reinterpret_cast<cudaStream_t>(stream));
  return run_ln_fwd(rows, h, dtype, x, 0, g, b, eps, y, mu, rstd,
                    reinterpret_cast<cudaStream_t>(stream));
}

size_t gptl_layernorm_bwd_scratch_bytes(int rows, int h) {
  (void)rows;
  return (size_t)3 * 512 * (size_t)(h > 0 ? h : 0) * sizeof(float);
}

int gptl_layernorm_bwd(int rows, int h, gptl_dtype dtype, const void *gy, const void *x,
                       const float *mu, const float *rstd, const void *g, const void *resid,
                       void *dx, float *dg, float *db, float *dx_sum, void *scratch,
                       gptl_stream_t stream) {
  if (!gy || !x || !mu || !rstd || !g || !resid || !dx || !dg || !db || !scratch) return GPTL_E_NULL;
  if (dtype != GPTL_FP16 && dtype != GPTL_BF16) return GPTL_E_DTYPE;
  if (!aligned16(gy) || !aligned16(x) || !aligned16(g) || !aligned16(resid) || !aligned16(dx) ||
      !aligned16(scratch))
    return GPTL_E_ALIGN;
  prof_start(reinterpret_cast<cudaStream_t>(stream));
  return run_ln_bwd(LNB_PARTS, rows, h, dtype, gy, x, mu, rstd, g, resid, dx, nullptr, dg, db,
                    dx_sum, nullptr,
                    static_cast<float *>(scratch), reinterpret_cast<cudaStream_t>(stream));
}

size_t gptl_colsum_scratch_bytes(int n, int groups) {
  if (n <= 0 || groups <= 0) return 0;
  return (size_t)kColsumMaxSplit * (size_t)n * (size_t)groups * sizeof(float);
}

int gptl_colsum(int rows, int n, int groups, long long ld, long long gstride, gptl_dtype dtype,
                const void *a, float *out, void *scratch, gptl_stream_t stream) {
  if (!a || !out || !scratch) return GPTL_E_NULL;
  if (dtype != GPTL_FP16 && dtype != GPTL_BF16) return GPTL_E_DTYPE;
  if (!aligned16(a) || !aligned16(scratch)) return GPTL_E_ALIGN;
  prof_start(reinterpret_cast<cudaStream_t>(stream));
  return run_colsum(rows, n, groups, ld, gstride, dtype, a, out, static_cast<float *>(scratch),
                    reinterpret_cast<cudaStream_t>(stream));
}

int gptl_attention_fwd(int batch, int seq, int hidden, int heads, int tp, gptl_dtype dtype,
                       const void *qkv, void *o, float *lse, gptl_stream_t stream) {
  if (!qkv || !o || !lse) return GPTL_E_NULL;
  if (dtype != GPTL_FP16 && dtype != GPTL_BF16) return GPTL_E_DTYPE;
  if (!aligned16(qkv) || !aligned16(o) || !aligned16(lse)) return GPTL_E_ALIGN;
  if (batch <= 0 || seq <= 0 || hidden <= 0 || heads <= 0 || tp <= 0) return GPTL_E_SHAPE;
  if (hidden % heads || heads % tp) return GPTL_E_SHAPE;
  GPTL_TRY(device_check());
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  prof_start(st);
  return run_attn_fwd(batch, seq, hidden / tp, heads / tp, tp, hidden / heads, dtype, qkv, o, lse, st);
}

int gptl_attention_bwd(int batch, int seq, int hidden, int heads, int tp, gptl_dtype dtype,
                       const void *qkv, const void *o, const void *dout, const float *lse,
                       float *dvec, void *dqkv, float *dbias_part, float *dbias,
                       gptl_stream_t stream) {
  if (!qkv || !o || !dout || !lse || !dvec || !dqkv) return GPTL_E_NULL;
  if ((dbias_part == nullptr) != (dbias == nullptr)) return GPTL_E_NULL;
  if (dbias && (!aligned16(dbias_part) || !aligned16(dbias))) return GPTL_E_ALIGN;
  if (dtype != GPTL_FP16 && dtype != GPTL_BF16) return GPTL_E_DTYPE;
  if (!aligned16(qkv) || !aligned16(o) || !aligned16(dout) || !aligned16(lse) || !aligned16(dvec) ||
      !aligned16(dqkv))
    return GPTL_E_ALIGN;
  if (batch <= 0 || seq <= 0 || hidden <= 0 || heads <= 0 || tp <= 0) return GPTL_E_SHAPE;
  if (hidden % heads || heads % tp) return GPTL_E_SHAPE;
  GPTL_TRY(device_check());
  const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int hs = hidden / tp, as = heads / tp, d = hidden / heads;
  if (d % 16 || d > 128 || seq % 16) return GPTL_E_SHAPE;
  prof_start(st);
  GPTL_TRY(run_attn_rowdot((long long)tp * batch * seq, seq, hs, as, d, dtype, dout, o, dvec, st));
  GPTL_TRY(run_attn_bwd(batch, seq, hs, as, tp, d, dtype, qkv, dout, lse, dvec, dqkv, dbias_part,
                        st));
  if (!dbias) return GPTL_OK;
  return launch_reduce_parts(dbias_part, batch * ((seq + 31) / 32), tp * 3 * hs, 1, dbias, nullptr,
                             nullptr, nullptr, st);
}

// Column sums with their partials in a fixed device array instead of
// caller memory (see gptl_colsum_noalloc in gptlayer_parts.h).
int gptl_colsum_noalloc(int rows, int n, int groups, long long ld, long long gstride,
                        gptl_dtype dtype, const void *a, float *out, gptl_stream_t stream) {
  if (!a || !out) return GPTL_E_NULL;
  if (dtype != GPTL_FP16 && dtype != GPTL_BF16) return GPTL_E_DTYPE;
  if (!aligned16(a)) return GPTL_E_ALIGN;
  if (rows <= 0 || n <= 0 || groups <= 0) return GPTL_E_SHAPE;
  if ((long long)n * groups > kNoAllocMaxWidth) return GPTL_E_TOO_LARGE;
  float *part = nullptr;
  GPTL_TRY(noalloc_scratch(&part));
  prof_start(reinterpret_cast<cudaStream_t>(stream));
  return run_colsum(rows, n, groups, ld, gstride, dtype, a, out, part,
                    reinterpret_cast<cudaStream_t>(stream));
}

// ------------------------------------------------------------- profiling
unsigned long long gptl_launch_count(void) { return g_launches; }

int gptl_profile_begin(int capacity) {
  if (capacity <= 0) return GPTL_E_ARG;
  if (g_prof.on) return GPTL_E_ARG;
  g_prof = Profiler();
  const int pool_n = 2 * capacity + 64;
  g_prof.pool = static_cast<cudaEvent_t *>(calloc((size_t)pool_n, sizeof(cudaEvent_t)));
  g_prof.recs = static_cast<ProfRec *>(calloc((size_t)capacity, sizeof(ProfRec)));
  if (!g_prof.pool || !g_prof.recs) {
    free(g_prof.pool);
    free(g_prof.recs);
    g_prof = Profiler();
    return GPTL_E_ARG;
  }
  for (int i = 0; i < pool_n; ++i) {
    if (cudaEventCreate(&g_prof.pool[i]) != cudaSuccess) {
      (void)cudaGetLastError();
      for (int j = 0; j < i; ++j) cudaEventDestroy(g_prof.pool[j]);
      free(g_prof.pool);
      free(g_prof.recs);
      g_prof = Profiler();
      return GPTL_E_CUDA;
    }
  }
  g_prof.pool_n = pool_n;
  g_prof.cap = capacity;
  g_prof.on = true;
  return GPTL_OK;
}

int gptl_profile_end(gptl_launch_record *out, int capacity, int *n_out, long long *dropped) {
  if (!g_prof.on) return GPTL_E_ARG;
  int rc = GPTL_OK;
  if (cudaDeviceSynchronize() != cudaSuccess) {
    (void)cudaGetLastError();
    rc = GPTL_E_CUDA;
  }
  int n = 0;
  for (int i = 0; i < g_prof.n && rc == GPTL_OK; ++i) {
    if (!out || n >= capacity) break;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, g_prof.recs[i].a, g_prof.recs[i].b) != cudaSuccess) {
      (void)cudaGetLastError();
      rc = GPTL_E_CUDA;
      break;
    }
    out[n].kind = g_prof.recs[i].kind;
    out[n].tag = g_prof.recs[i].tag;
    out[n].ms = ms;
    ++n;
  }
  if (n_out) *n_out = n;
  if (dropped) *dropped = g_prof.dropped + (g_prof.n - n);
  for (int i = 0; i < g_prof.pool_n; ++i) cudaEventDestroy(g_prof.pool[i]);
  free(g_prof.pool);
  free(g_prof.recs);
  g_prof = Profiler();
  return rc;
}

const char *gptl_tag_name(int tag) {
  switch (tag) {
    case GPTL_TAG_NONE: return "-";
    case GPTL_TAG_F1_LN1: return "F1 ln1";
    case GPTL_TAG_F2_QKV: return "F2 qkv";
    case GPTL_TAG_F3_F5_ATTN: return "F3-F5 attention";
    case GPTL_TAG_F6_OUTPROJ: return "F6 outproj";
    case GPTL_TAG_F7_LN2: return "F7 ln2";
    case GPTL_TAG_F8_FFN1_GELU: return "F8/F9 ffn1+gelu";
    case GPTL_TAG_F10_FFN2: return "F10 ffn2";
    case GPTL_TAG_B1_B3_DZ: return "B1/B3 dz";
    case GPTL_TAG_B2_DW2: return "B2 dw2";
    case GPTL_TAG_B2_DB2: return "B2 db2";
    case GPTL_TAG_B3_DB1: return "B3 db1";
    case GPTL_TAG_B4_DL2: return "B4 dl2";
    case GPTL_TAG_B5_DW1: return "B5 dw1";
    case GPTL_TAG_B6_LN2: return "B6 ln2 bwd";
    case GPTL_TAG_B7_DWO: return "B7 dwo";
    case GPTL_TAG_B7_DO: return "B7 do";
    case GPTL_TAG_B8_B10_ATTN: return "B8-B10 attention bwd";
    case GPTL_TAG_B9_ROWDOT: return "B9 rowdot";
    case GPTL_TAG_B11_DBQKV: return "B11 dbqkv";
    case GPTL_TAG_B11_DWQKV: return "B11 dwqkv";
    case GPTL_TAG_B11_DL1: return "B11 dl1";
    case GPTL_TAG_B12_LN1: return "B12 ln1 bwd";
    case GPTL_TAG_B0_WT: return "B0 weights^T";
    case GPTL_TAG_B2_DOUT_T: return "B2 dOut^T";
    case GPTL_TAG_B5_L2_T: return "B5 L2^T";
    case GPTL_TAG_B7_DH_T: return "B7 dH^T";
    case GPTL_TAG_B11_L1_T: return "B11 L1^T";
    case GPTL_TAG_O1_OVERFLOW: return "O1 overflow";
    case GPTL_TAG_O2_ADAM: return "O2 adam";
    case GPTL_TAG_O3_SCALE: return "O3 scale";
    default: return "?";
  }
}

}  // extern "C"
