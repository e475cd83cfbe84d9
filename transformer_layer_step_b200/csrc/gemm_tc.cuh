// gemm_tc.cuh — persistent tcgen05/TMEM GEMM for sm_100a, fed by TMA.
//
// One kernel serves every dense contraction of the layer step outside
// attention: the four linear layers (forward, input gradient, weight
// gradient).  D[M,N] = sum_k A[M,k] * B[N,k] per group, with
//   * operands read through 3-D TMA views (x = contiguous column, row, group)
//     and staged in 128- or 256-row / BN-row x 64-deep shared-memory tiles;
//   * either operand K-major (rows = M/N index, x = K) or MN-major
//     (rows = K index, x = M/N), using the hardware transpose of the MMA
//     instead of any transposing copy;
//   * an optional walk of the K loop over tensor-parallel shards (the row
//     split's partial sums and the column split's input-gradient sums are
//     accumulated in one TMEM accumulator: "Megatron-LM 3D parallelism" §1
//     describes the all-reduce this replaces);
//   * fused epilogues: bias, residual, bias+GeLU (writes Z and GeLU(Z): the
//     fused_bias_gelu of "Training GPT-2 with Megatron-LM" §6.2), GeLU'
//     scaling of an input gradient (optionally writing GeLU of its stored
//     argument again: the activation recomputed for the weight gradient),
//     32-row column sums of a 16-bit output (a bias gradient's partial
//     sums), fp32 weight-gradient store;
//   * outputs leave through shared memory with TMA tensor stores: each
//     epilogue warp stages 32-row x 64-byte boxes (64B swizzle) and one lane
//     stores them, so global writes are whole 32-byte sectors and the ragged
//     M/N edges are clipped by the tensor map.
//
// Warp roles (384 threads, one CTA per SM): two pipelines, each a TMA
// producer warp (0, 2), an MMA warp (1, 3) whose one thread issues
// tcgen05.mma (M=128, N=BN, K=16 each) and a TMEM accumulator of BN columns;
// warp 1 allocates the 512 TMEM columns.  Warps 4..11 drain accumulators with
// tcgen05.ld: a warp may only read the TMEM lane quarter (warp % 4), so two
// epilogue warps share each quarter and split its columns in half.  How the
// pipelines share the work (alternating tiles, K halves of each tile, or
// 256-row tiles split by M) is described at gemm_tc_kernel.
#pragma once
#include "common.cuh"

namespace gptl {

constexpr int kBM = 128;          // tile rows (UMMA M)
constexpr int kBK = 64;           // tile depth per pipeline stage
constexpr int kGemmThreads = 384;
constexpr int kEpiWarps = 8;
// registers per thread: the launch allocation (one CTA per SM at 384 threads
// gets 168 each) and the split by role after setup.  The TMA / MMA warpgroup
// gives registers up and the two epilogue warpgroups take them; the split
// must add up to the launch allocation exactly, or the increase never
// completes, so the host checks the compiled count before the first launch.
constexpr int kGemmRegs = 168;
constexpr int kRoleRegs = 56;
constexpr int kEpiRegs = 224;
static_assert(128 * kRoleRegs + 256 * kEpiRegs == kGemmThreads * kGemmRegs, "register split");

enum : int { kActNone = 0, kActGelu = 1, kActDGelu = 2 };

constexpr int kStageBoxBytes = 2048;                 // one 32-row x 64-byte store box
constexpr int kStagingBytes = 8 * 2 * kStageBoxBytes;  // two boxes per epilogue warp

struct OperandRule {
  int mn_major;                // 0: K-major, 1: MN-major
  int w;                       // MN-major chunk width in elements (64, 32 or 16)
  int x_mod, x_mul, x_off;     // column offset of group G: (G % x_mod) * x_mul + x_off
  int g_div;                   // group coordinate G / g_div ...
  int k_shard;                 // ... plus the k-shard index when set
};

struct alignas(64) GemmParams {
  CUtensorMap map_a;
  CUtensorMap map_b;
  CUtensorMap map_o;           // output, or the split-K partials; box {64 B / elem, 32, 1, 1}
  CUtensorMap map_o2;          // GeLU(Z) when act == GELU
  OperandRule ra, rb;
  int M, N, K, groups, k_shards;
  int split;                   // K slices per tile (split-K); 1 = none
  int pipe_k;                  // 1: both pipelines work on every tile, one K half each
  int m2;                      // 1: 256-row tiles, one M half per pipeline, one shared ring
  float *ws;                   // split-K partials [split][groups][M][N] fp32
  long long ws_slice;          // groups * M * N
  int bn, bn_alloc, stages, tmem_cols;
  uint32_t idesc;
  int m_tiles, n_tiles;
  int band;                    // tile order: bands of `band` N tiles, M tiles fastest in a band
  long long total_tiles;
  // epilogue
  int o_mod;                   // output group G at map coordinates (G % o_mod, G / o_mod), or
  int o_flat;                  // (G, 0) when o_flat is set
  int out_f32;
  const void *bias;
  long long bias_g_stride;
  const void *resid;
  long long ld_resid;
  int resid_f32;
  const void *aux;             // GeLU' argument, same layout as the output
  long long ldo;
  long long o_str_mod, o_str_div;
  int act;
  int write_o2;                // GELU: GeLU(value) to map_o2; DGELU: GeLU(aux) to map_o2
  int *nonfinite;              // fp32 outputs: set to 1 if any value written is inf or NaN
  float *colsum;               // 16-bit outputs: 32-row column sums [colsum_rows][groups][N]
  int colsum_rows;             // ceil(M / 32)
  int out_evict_first;         // store the output with L2 evict-first priority
};

// true when an fp32 value is inf or NaN (all exponent bits set)
__device__ __forceinline__ bool not_finite(float v) { return !(fabsf(v) <= 3.402823466e38f); }

struct TileInfo {
  int g, m0, n0, kb_begin, kb_end, slice;
};

__device__ __forceinline__ TileInfo tile_info(const GemmParams &p, long long idx) {
  TileInfo t;
  const long long tile = idx / p.split;
  t.slice = (int)(idx - tile * p.split);
  const long long tpg = (long long)p.m_tiles * p.n_tiles;
  t.g = (int)(tile / tpg);
  const int rem = (int)(tile - (long long)t.g * tpg);
  // the tiles of a band of N columns in M order: the CTAs working at the same
  // time read the same k-slabs of B (the weights, in most products) from L2,
  // instead of each streaming a B tile that the other M rows need later
  const int span = p.m_tiles * p.band;
  const int bnd = rem / span, r2 = rem - bnd * span;
  const int mt = r2 % p.m_tiles, nt = bnd * p.band + r2 / p.m_tiles;
  t.m0 = mt * (p.m2 ? 2 * kBM : kBM);
  t.n0 = nt * p.bn;
  t.kb_begin = 0;
  t.kb_end = (p.K + kBK - 1) / kBK;
  if (p.split > 1) {           // balanced slices, none empty while split <= k-blocks
    const int nkb = t.kb_end - t.kb_begin, b = t.kb_begin;
    t.kb_begin = b + (int)((long long)t.slice * nkb / p.split);
    t.kb_end = b + (int)((long long)(t.slice + 1) * nkb / p.split);
  }
  return t;
}

__device__ __forceinline__ uint32_t swizzle_layout(int w) {
  return w == 64 ? 2u : (w == 32 ? 4u : 6u);
}

// Issue the TMA loads of one operand tile for k-block starting at k0.
__device__ __forceinline__ void load_operand(const CUtensorMap *map, const OperandRule &r,
                                             uint32_t dst, int rows, int g, int ks, int mn0,
                                             int k0, uint32_t bar) {
  const int x0 = (g % r.x_mod) * r.x_mul + r.x_off;
  const int gc = g / r.g_div + (r.k_shard ? ks : 0);
  if (!r.mn_major) {
    tma_load_3d(dst, map, x0 + k0, mn0, gc, bar);
  } else {
    const int chunks = rows / r.w;
    for (int c = 0; c < chunks; ++c)
      tma_load_3d(dst + (uint32_t)(c * kBK * r.w * 2), map, x0 + mn0 + c * r.w, k0, gc, bar);
  }
}

// Shared-memory descriptor of the 16-deep slice `step` of an operand tile.
//   K-major tile  [rows][64] (128B rows, 128B swizzle): SBO = 8 rows = 1024 B,
//                 the slice starts 32 B further per step.
//   MN-major tile [rows/w chunks][64 k-rows][w]: rows of 2w bytes, SBO = 8
//                 k-rows = 16w B, LBO = chunk stride = 64 * 2w B; the slice
//                 starts 16 k-rows further per step.
__device__ __forceinline__ uint64_t operand_desc(const OperandRule &r, uint32_t base, int step) {
  if (!r.mn_major) return make_smem_desc(base + (uint32_t)step * 32u, 16u, 1024u, 2u);
  const uint32_t row_b = (uint32_t)r.w * 2u;
  return make_smem_desc(base + (uint32_t)step * 16u * row_b, (uint32_t)kBK * row_b, 8u * row_b,
                        swizzle_layout(r.w));
}

// Global inputs of one 16-column epilogue chunk, loaded one chunk ahead so
// that their latency overlaps the previous chunk's arithmetic.
struct EpiIn {
  uint4 bias[2];     // 16-bit bias
  uint4 v[4];        // fp32 residual (4 vectors), or 16-bit residual / GeLU' argument (2):
                     // a GEMM has at most one of them
};

// Per-thread row pointers of the epilogue inputs for one tile (null when
// unused or when the row is past M).
struct EpiRow {
  const uint8_t *bias;
  const uint8_t *resid;
  const uint8_t *aux;
  bool row_ok;                 // the row is inside M
};

template <typename T>
__device__ __forceinline__ EpiRow epilogue_row(const GemmParams &p, int g, int row) {
  EpiRow e{nullptr, nullptr, nullptr, row < p.M};
  if (p.split > 1 || row >= p.M) return e;
  if (p.bias) e.bias = reinterpret_cast<const uint8_t *>(static_cast<const T *>(p.bias) +
                                                        (long long)g * p.bias_g_stride);
  if (p.resid)
    e.resid = static_cast<const uint8_t *>(p.resid) +
              (long long)row * p.ld_resid * (p.resid_f32 ? 4 : (int)sizeof(T));
  if (p.act == kActDGelu)
    e.aux = reinterpret_cast<const uint8_t *>(
        static_cast<const T *>(p.aux) + (long long)(g % p.o_mod) * p.o_str_mod +
        (long long)(g / p.o_mod) * p.o_str_div + (long long)row * p.ldo);
  return e;
}

template <typename T>
__device__ __forceinline__ void epilogue_load(const GemmParams &p, const EpiRow &e, int n, EpiIn &in) {
  if (e.bias) {
    const uint4 *b = reinterpret_cast<const uint4 *>(e.bias) + n / 8;
    in.bias[0] = __ldg(b);
    in.bias[1] = __ldg(b + 1);
  }
  if (e.resid) {
    if (p.resid_f32) {
      const uint4 *rr = reinterpret_cast<const uint4 *>(e.resid) + n / 4;
#pragma unroll
      for (int q = 0; q < 4; ++q) in.v[q] = rr[q];
    } else {
      const uint4 *rr = reinterpret_cast<const uint4 *>(e.resid) + n / 8;
      in.v[0] = rr[0];
      in.v[1] = rr[1];
    }
  } else if (e.aux) {
    const uint4 *xp = reinterpret_cast<const uint4 *>(e.aux) + n / 8;
    in.v[0] = xp[0];
    in.v[1] = xp[1];
  }
}

// Shared address of 16-byte piece j (0..3) of row r in a 32-row x 64-byte
// staging box laid out with the 64B swizzle of the store's tensor map.
__device__ __forceinline__ uint32_t box_piece(uint32_t box, int r, int j) {
  return box + (uint32_t)(r * 64) + (uint32_t)((j ^ ((r >> 1) & 3)) << 4);
}

// Finish one 16-column chunk (fp32 accumulator values r) and write it into
// the staging box(es): 16-bit outputs fill half a box (pieces 2*slot,
// 2*slot+1), fp32 outputs a whole box.  With p.colsum, the warp also sums the
// chunk's 16 columns as stored (rounded; rows past M count 0) over its 32
// rows and writes the sums to cs_out[0..15] (when cs_out is not null).
template <typename T, bool CS>
__device__ __forceinline__ void epilogue_chunk(const GemmParams &p, const EpiRow &e,
                                               const uint32_t (&r)[16], const EpiIn &in,
                                               uint32_t box, uint32_t box2, int lane, int slot,
                                               bool &bad, float *cs_out) {
  float v[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  if (e.bias) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float f[8];
      unpack8<T>(in.bias[h], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[8 * h + i] += f[i];
    }
  }
  if (e.resid) {
    if (p.resid_f32) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[4 * q] += __uint_as_float(in.v[q].x); v[4 * q + 1] += __uint_as_float(in.v[q].y);
        v[4 * q + 2] += __uint_as_float(in.v[q].z); v[4 * q + 3] += __uint_as_float(in.v[q].w);
      }
    } else {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float f[8];
        unpack8<T>(in.v[h], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[8 * h + i] += f[i];
      }
    }
  }
  if (p.out_f32 || p.split > 1) {
    if (p.nonfinite && p.split == 1 && e.row_ok) {   // split-K: checked on the final sums
#pragma unroll
      for (int i = 0; i < 16; ++i) bad |= not_finite(v[i]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
      st_shared_v4(box_piece(box, lane, j),
                   make_uint4(__float_as_uint(v[4 * j]), __float_as_uint(v[4 * j + 1]),
                              __float_as_uint(v[4 * j + 2]), __float_as_uint(v[4 * j + 3])));
    return;
  }
  if (p.act == kActGelu) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float z[8], a[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) z[i] = v[8 * h + i];
      const uint4 zq = pack8<T>(z);
      float zr[8];
      unpack8<T>(zq, zr);                 // GeLU of the stored (rounded) Z
#pragma unroll
      for (int i = 0; i < 8; ++i) a[i] = gelu_f(zr[i]);
      st_shared_v4(box_piece(box, lane, 2 * slot + h), zq);
      st_shared_v4(box_piece(box2, lane, 2 * slot + h), pack8<T>(a));
    }
    return;
  }
  if (e.aux) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float z[8], a[8];
      unpack8<T>(in.v[h], z);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[8 * h + i] *= gelu_prime_f(z[i]);
      if (p.write_o2) {               // the activation, recomputed from its stored argument
#pragma unroll
        for (int i = 0; i < 8; ++i) a[i] = gelu_f(z[i]);
        st_shared_v4(box_piece(box2, lane, 2 * slot + h), pack8<T>(a));
      }
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float f[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = v[8 * h + i];
    const uint4 pk = pack8<T>(f);
    st_shared_v4(box_piece(box, lane, 2 * slot + h), pk);
    if constexpr (CS) {                 // the stored values, for the column sums
      unpack8<T>(pk, f);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[8 * h + i] = e.row_ok ? f[i] : 0.f;
    }
  }
  if constexpr (CS) {
    const float sum = warp_colsum16(v, lane);
    if (cs_out && (lane & 1) == 0) cs_out[(lane >> 1) & 15] = sum;
  }
}

// Two independent pipelines share the CTA.  Either the CTA's tiles alternate
// between them (local tile t goes to pipeline t % 2), or, with pipe_k (few,
// long-K tiles), both work on every tile: pipeline p reduces the p-th half of
// the tile's k-blocks into its own accumulator and the epilogue adds the two
// (acc0 + acc1, a fixed order).  Each pipeline has its own
// producer warp, shared-memory ring (p.stages stages), MMA-issuing warp and
// TMEM accumulator (columns [pipe * bn_alloc, +bn)).  Measured on B200, one
// thread's stream of tcgen05.mma instructions runs at a fixed rate per
// instruction well below the tensor core's, and two issuing warps run
// concurrently; the two accumulators also give the epilogue of one tile the
// other pipeline's MMAs to overlap with.
// Does pipeline pp take local tile t, and which of its k-blocks?
__device__ __forceinline__ bool pipe_takes(const GemmParams &p, int t, int pp) {
  return (p.pipe_k || p.m2) ? true : ((t & 1) == pp);
}
__device__ __forceinline__ void pipe_kb_range(const GemmParams &p, const TileInfo &ti, int pp,
                                              int &kb0, int &kb1) {
  kb0 = ti.kb_begin;
  kb1 = ti.kb_end;
  if (p.pipe_k) {
    const int mid = ti.kb_begin + (ti.kb_end - ti.kb_begin) / 2;
    if (pp == 0) kb1 = mid;
    else kb0 = mid;
  }
}

// CS: the instantiation with the epilogue's column sums (p.colsum set); the
// others carry no code for them (measured: that code alone slowed every
// short-K product at the GPT-2 117M shape by 3-10 %).
template <typename T, bool CS>
__global__ void __launch_bounds__(kGemmThreads, 1) gemm_tc_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int a_rows = p.m2 ? 2 * kBM : kBM;
  const int a_bytes = a_rows * kBK * 2;
  const int b_bytes = p.bn * kBK * 2;
  const int stage_bytes = a_bytes + b_bytes;
  const int S = p.stages;                                   // stages per ring
  const int rings = p.m2 ? 1 : 2;                           // m2: one ring both pipelines read
  const uint32_t staging_s = smem_u32(smem + rings * S * stage_bytes);   // 1024-aligned
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + rings * S * stage_bytes + kStagingBytes);
  // bars: full[pipe][S] empty[pipe][S] tfull[2] tempty[2] drain[2]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 4 * S + 6);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t tiles_s = smem_u32(smem);
  auto full_bar = [&](int pp, int s) { return smem_u32(&bars[pp * S + s]); };
  auto empty_bar = [&](int pp, int s) { return smem_u32(&bars[2 * S + pp * S + s]); };
  auto tfull_bar = [&](int pp) { return smem_u32(&bars[4 * S + pp]); };
  auto tempty_bar = [&](int pp) { return smem_u32(&bars[4 * S + 2 + pp]); };
  auto drain_bar = [&](int pp) { return smem_u32(&bars[4 * S + 4 + pp]); };
  auto stage_addr = [&](int pp, int s) { return tiles_s + (uint32_t)((pp * S + s) * stage_bytes); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int pp = 0; pp < 2; ++pp) {
      for (int s = 0; s < S; ++s) {
        mbar_init(full_bar(pp, s), 1);
        mbar_init(empty_bar(pp, s), p.m2 ? 2 : 1);   // m2: both MMA warps release a stage
      }
      mbar_init(tfull_bar(pp), 1);
      mbar_init(tempty_bar(pp), kEpiWarps);
      mbar_init(drain_bar(pp), 1);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.map_a);
    prefetch_tensormap(&p.map_b);
    prefetch_tensormap(&p.map_o);
    if (p.write_o2) prefetch_tensormap(&p.map_o2);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // registers by role: the TMA / MMA warps (warpgroup 0) need few, the
  // epilogue warps (warpgroups 1, 2) hold four accumulator chunks in flight
  if (warp < 4) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;\n" ::"n"(kRoleRegs) : "memory");
  else asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;\n" ::"n"(kEpiRegs) : "memory");

  if (warp < 4) {
    const int pp = warp >> 1;                 // pipeline of this warp
    const bool producer_warp = (warp & 1) == 0;
    // m2: the one shared ring is filled by pipeline 0's producer alone
    if (lane == 0 && producer_warp && !(p.m2 && pp == 1)) {
      // ------------------------------------------------ TMA producer
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity = 0;
      int t = 0;                              // local tile counter
      for (long long idx = blockIdx.x; idx < p.total_tiles; idx += gridDim.x) {
        const TileInfo ti = tile_info(p, idx);
        if (!pipe_takes(p, t++, pp)) continue;
        int kb0, kb1;
        pipe_kb_range(p, ti, pp, kb0, kb1);
        for (int ks = 0; ks < p.k_shards; ++ks)
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(empty_bar(pp, stage), phase ^ 1, abort_flag)) goto producer_abort;
            const uint32_t fb = full_bar(pp, stage);
            mbar_arrive_expect_tx(fb, (uint32_t)stage_bytes);
            const uint32_t sa = stage_addr(pp, stage);
            load_operand(&p.map_a, p.ra, sa, a_rows, ti.g, ks, ti.m0, kb * kBK, fb);
            load_operand(&p.map_b, p.rb, sa + a_bytes, p.bn, ti.g, ks, ti.n0, kb * kBK, fb);
            issued |= 1u << stage;
            parity = (parity & ~(1u << stage)) | (phase << stage);
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
            }
          }
      }
      goto producer_done;
    producer_abort:
      // let our own copies land before the CTA exits
      for (int s = 0; s < S; ++s)
        if (issued & (1u << s)) mbar_wait_drain(full_bar(pp, s), (parity >> s) & 1u);
    producer_done:;
    } else if (lane == 0 && !producer_warp) {
      // ------------------------------------------------ MMA issuer
      int stage = 0;
      uint32_t phase = 0, acc_phase = 0;
      int t = 0;
      const uint32_t d_tmem = tmem_base + (uint32_t)(pp * p.bn_alloc);
      const int ring = p.m2 ? 0 : pp;
      for (long long idx = blockIdx.x; idx < p.total_tiles; idx += gridDim.x) {
        const TileInfo ti = tile_info(p, idx);
        if (!pipe_takes(p, t++, pp)) continue;
        if (!mbar_wait(tempty_bar(pp), acc_phase ^ 1, abort_flag)) goto mma_abort;
        tc_fence_after();
        int kb0, kb1;
        pipe_kb_range(p, ti, pp, kb0, kb1);
        int it = 0;
        for (int ks = 0; ks < p.k_shards; ++ks)
          for (int kb = kb0; kb < kb1; ++kb) {
            if (!mbar_wait(full_bar(ring, stage), phase, abort_flag)) goto mma_abort;
            tc_fence_after();
            // m2: this pipeline's 128 rows of the 256-row A tile (K-major rows,
            // or MN-major column chunks: 16 KB into the tile either way)
            const uint32_t sa = stage_addr(ring, stage) + (p.m2 ? (uint32_t)(pp * kBM * kBK * 2) : 0u);
            const uint32_t sb = stage_addr(ring, stage) + (uint32_t)a_bytes;
            const int nsteps = min(kBK, p.K - kb * kBK) / 16;
            for (int s = 0; s < nsteps; ++s)
              tc_mma_f16(d_tmem, operand_desc(p.ra, sa, s), operand_desc(p.rb, sb, s), p.idesc,
                         (it > 0 || s > 0) ? 1u : 0u);
            tc_commit(empty_bar(ring, stage));
            ++it;
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
            }
          }
        tc_commit(tfull_bar(pp));
        acc_phase ^= 1;
      }
      goto mma_done;
    mma_abort:
      // wait for the MMAs already issued before TMEM is released
      tc_commit(drain_bar(pp));
      mbar_wait_drain(drain_bar(pp), 0);
    mma_done:;
    }
  } else {
    // -------------------------------------------------- epilogue warps
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - 4) >> 2;        // which half of the tile's columns
    const bool wide = p.out_f32 || p.split > 1;     // fp32: one chunk per box
    const bool two = !wide && p.write_o2;     // a second output: both boxes per chunk pair
    // no bias, residual, activation or second K half: nothing to load per chunk
    const bool grouped = !CS && !p.bias && !p.resid && p.act == kActNone && !p.pipe_k;
    const uint32_t my_boxes = staging_s + (uint32_t)((warp - 4) * 2 * kStageBoxBytes);
    int box_i = 0;                           // boxes issued by this warp (selects the buffer)
    bool bad = false;                        // an fp32 output value was inf or NaN
    uint32_t acc_phase[2] = {0u, 0u};
    int t = 0;
    for (long long idx = blockIdx.x; idx < p.total_tiles; idx += gridDim.x) {
      const TileInfo ti = tile_info(p, idx);
      // accumulator of this tile; with pipe_k or m2 both are (pp = 0 and 1)
      const bool both = p.pipe_k || p.m2;
      const int pp = both ? 0 : (t & 1);
      ++t;
      bool got = mbar_wait(tfull_bar(pp), acc_phase[pp], abort_flag);
      if (got && both) got = mbar_wait(tfull_bar(1), acc_phase[1], abort_flag);
      if (!got) break;
      acc_phase[pp] ^= 1;
      if (both) acc_phase[1] ^= 1;
      tc_fence_after();
      for (int hf = 0; hf < (p.m2 ? 2 : 1); ++hf) {   // m2: the tile's two 128-row halves
      const int row0 = ti.m0 + hf * kBM + q * 32;
      const EpiRow er = epilogue_row<T>(p, ti.g, row0 + lane);
      const uint32_t t_row =
          tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)((pp + hf) * p.bn_alloc);
      // output map coordinates of this tile's group
      int oz, ow;
      if (p.split > 1) { oz = ti.slice * p.groups + ti.g; ow = 0; }
      else if (p.o_flat) { oz = ti.g; ow = 0; }
      else { oz = ti.g % p.o_mod; ow = ti.g / p.o_mod; }
      // this warp's 16-column chunks [c0, c1); the halves split at an even
      // chunk so that a 16-bit box (two chunks) never straddles them
      const int nchunk = p.bn / 16;
      const int csplit = 2 * ((nchunk + 3) / 4);
      const int c0 = half ? csplit : 0;
      int c1 = half ? nchunk : csplit;
      const int valid = (p.N - ti.n0 + 15) / 16;   // chunks inside N
      if (c1 > valid) c1 = valid;
      uint32_t ra[16], rb[16];
      EpiIn ia, ib;
      const uint32_t t_row2 = t_row + (uint32_t)p.bn_alloc;   // pipe_k: the second K half
      auto ld = [&](int c, uint32_t (&r)[16]) { tmem_ld16(t_row + (uint32_t)(c * 16), r); };
      // pipe_k: add the second accumulator's chunk c (loaded here, not ahead)
      auto sum2 = [&](int c, uint32_t (&r)[16]) {
        if (p.pipe_k) {
          uint32_t r2[16];
          tmem_ld16(t_row2 + (uint32_t)(c * 16), r2);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) + __uint_as_float(r2[i]));
        }
      };
      auto process = [&](int c, const uint32_t (&r)[16], const EpiIn &in) {
        const int slot = wide ? 0 : ((c - c0) & 1);
        const bool first = slot == 0, last = wide || slot == 1 || c + 1 == c1;
        const uint32_t buf = my_boxes + (uint32_t)((two ? 0 : (box_i & 1)) * kStageBoxBytes);
        if (first) {                         // the box buffer(s) must be free again
          if (lane == 0) {
            if (two) bulk_wait_read<0>();
            else bulk_wait_read<1>();
          }
          __syncwarp();
        }
        // this warp's 32 rows form partial row row0 / 32 of the column sums
        float *cs_out = nullptr;
        if (CS && (row0 >> 5) < p.colsum_rows)
          cs_out = p.colsum + ((long long)(row0 >> 5) * p.groups + ti.g) * p.N + ti.n0 + c * 16;
        epilogue_chunk<T, CS>(p, er, r, in, buf, my_boxes + kStageBoxBytes, lane, slot, bad, cs_out);
        if (last) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int x = ti.n0 + (c - slot) * 16;
            if (p.out_evict_first) tma_store_4d_hint(&p.map_o, buf, x, row0, oz, ow, l2_policy_evict_first());
            else tma_store_4d(&p.map_o, buf, x, row0, oz, ow);
            if (two) tma_store_4d(&p.map_o2, my_boxes + kStageBoxBytes, x, row0, oz, ow);
            bulk_commit();
          }
          ++box_i;
        }
      };
      if (grouped) {
        // the grouped path's chunk: the accumulator values go to the box as
        // they are (fp32) or rounded to 16 bits, with no epilogue arithmetic
        auto process_plain = [&](int c, const uint32_t (&r)[16]) {
          const int slot = wide ? 0 : ((c - c0) & 1);
          const bool first = slot == 0, last = wide || slot == 1 || c + 1 == c1;
          const uint32_t buf = my_boxes + (uint32_t)((box_i & 1) * kStageBoxBytes);
          if (first) {
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
          }
          if (wide) {
            if (p.nonfinite && p.split == 1 && er.row_ok) {
#pragma unroll
              for (int i = 0; i < 16; ++i) bad |= not_finite(__uint_as_float(r[i]));
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              st_shared_v4(box_piece(buf, lane, j), make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]));
          } else {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float f[8];
#pragma unroll
              for (int i = 0; i < 8; ++i) f[i] = __uint_as_float(r[8 * h + i]);
              st_shared_v4(box_piece(buf, lane, 2 * slot + h), pack8<T>(f));
            }
          }
          if (last) {
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              const int x = ti.n0 + (c - slot) * 16;
              if (p.out_evict_first) tma_store_4d_hint(&p.map_o, buf, x, row0, oz, ow, l2_policy_evict_first());
              else tma_store_4d(&p.map_o, buf, x, row0, oz, ow);
              bulk_commit();
            }
            ++box_i;
          }
        };
        // four chunks' tensor-memory loads in flight before one wait: the
        // load latency, which bounds this epilogue, is paid once per 64 columns
        for (int c = c0; c < c1; c += 4) {
          uint32_t rg[4][16];
#pragma unroll
          for (int g = 0; g < 4; ++g)
            if (c + g < c1) ld(c + g, rg[g]);
          tmem_wait_ld();
#pragma unroll
          for (int g = 0; g < 4; ++g)
            if (c + g < c1) process_plain(c + g, rg[g]);
        }
        continue;
      }
      // with epilogue inputs: the load of chunk c+1 (and its inputs) is in
      // flight while chunk c is processed (tcgen05.wait::ld waits for every
      // earlier load)
      if (c0 < c1) {
        ld(c0, ra);
        epilogue_load<T>(p, er, ti.n0 + c0 * 16, ia);
        tmem_wait_ld();
        sum2(c0, ra);
      }
      for (int c = c0; c < c1; c += 2) {
        const bool has_b = c + 1 < c1;
        if (has_b) {
          ld(c + 1, rb);
          epilogue_load<T>(p, er, ti.n0 + (c + 1) * 16, ib);
        }
        process(c, ra, ia);
        tmem_wait_ld();
        if (!has_b) break;
        sum2(c + 1, rb);
        const bool has_a = c + 2 < c1;
        if (has_a) {
          ld(c + 2, ra);
          epilogue_load<T>(p, er, ti.n0 + (c + 2) * 16, ia);
        }
        process(c + 1, rb, ib);
        tmem_wait_ld();
        if (has_a) sum2(c + 2, ra);
      }
      }   // halves
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(tempty_bar(pp));
        if (both) mbar_arrive(tempty_bar(1));
      }
    }
    if (p.nonfinite && __any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.nonfinite, 1);
    // the staged boxes must be read, and the stores done, before the CTA exits
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, (uint32_t)p.tmem_cols);
  }
}

// out[G](m, n) = sum over s < split of ws[s][G][m][n], in slice order, into
// the strided fp32 output of the GEMM; 4 columns per thread.  With
// `nonfinite`, any inf or NaN sum sets it to 1.
__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float *__restrict__ ws,
                                                           long long ws_slice, int split, int M,
                                                           int N, int groups, float *out,
                                                           long long ldo, int o_mod,
                                                           long long o_str_mod,
                                                           long long o_str_div, int *nonfinite) {
  const long long n4 = ws_slice / 4;
  bool bad = false;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (long long)gridDim.x * blockDim.x) {
    const long long e = i * 4;
    const int g = (int)(e / ((long long)M * N));
    const long long rem = e - (long long)g * M * N;
    const int m = (int)(rem / N), n = (int)(rem - (long long)(rem / N) * N);
    float4 acc = reinterpret_cast<const float4 *>(ws)[i];
    for (int s = 1; s < split; ++s) {
      const float4 v = reinterpret_cast<const float4 *>(ws + (long long)s * ws_slice)[i];
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    const long long off = (long long)(g % o_mod) * o_str_mod + (long long)(g / o_mod) * o_str_div +
                          (long long)m * ldo + n;
    *reinterpret_cast<float4 *>(out + off) = acc;
    bad |= not_finite(acc.x) | not_finite(acc.y) | not_finite(acc.z) | not_finite(acc.w);
  }
  if (nonfinite && __any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0) atomicOr(nonfinite, 1);
}

// Row term of the softmax backward: D[g][p] = sum_c dO[p][c] * O[p][c] over
// the head's d columns (equal to sum_q P[p][q] dP[p][q], since O = P V).
// A block takes 8 rows of the [t*b*s][h/t] matrices and walks them in chunks
// of whole heads (at most kRowdotChunkVec 16-byte vectors per row): a warp per
// row reads the chunk in coalesced vectors and leaves one partial dot per
// vector in shared memory; then one thread per (row, head of the chunk) adds
// the head's d/8 partials in order.  Any row width and number of heads.
constexpr int kRowdotChunkVec = 512;
template <typename T>
__global__ void __launch_bounds__(256) attn_rowdot_kernel(const T *__restrict__ dout,
                                                          const T *__restrict__ o, float *__restrict__ dvec,
                                                          long long rows, int s, int hs, int as,
                                                          int d) {
  __shared__ float part[8][kRowdotChunkVec];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r0 = (long long)blockIdx.x * 8;
  const long long r = r0 + w;
  const int vh = d / 8;                        // vectors per head
  const int hpc = kRowdotChunkVec / vh;        // whole heads per chunk
  for (int h0 = 0; h0 < as; h0 += hpc) {
    const int nh = min(hpc, as - h0);
    const int nv = nh * vh;
    if (r < rows) {
      const uint4 *a = reinterpret_cast<const uint4 *>(dout + r * hs) + h0 * vh;
      const uint4 *b = reinterpret_cast<const uint4 *>(o + r * hs) + h0 * vh;
      for (int v = lane; v < nv; v += 32) {
        float fa[8], fb[8];
        unpack8<T>(__ldcs(a + v), fa);
        unpack8<T>(__ldcs(b + v), fb);
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(fa[e], fb[e], acc);
        part[w][v] = acc;
      }
    }
    __syncthreads();
    for (int i = threadIdx.x; i < 8 * nh; i += blockDim.x) {
      const int rl = i / nh, hc = i - rl * nh;    // (row in block, head in chunk)
      const long long rr = r0 + rl;
      if (rr < rows) {
        float acc = 0.f;
        for (int v = 0; v < vh; ++v) acc += part[rl][hc * vh + v];
        const long long zb = rr / s, pos = rr - zb * s;
        dvec[(zb * as + h0 + hc) * s + pos] = acc;
      }
    }
    __syncthreads();
  }
}

}  // namespace gptl
