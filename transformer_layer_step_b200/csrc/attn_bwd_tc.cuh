// attn_bwd_tc.cuh — fused causal attention backward on tcgen05 (sm_100a).
//
// The backward of the fused scale-mask-softmax attention ("Training GPT-2
// with Megatron-LM" §6.2) without materialising P or dS in HBM.  P is
// recomputed from the scores and each query row's base-2 log-sum-exp saved
// by the forward; the softmax backward's row term D = dO . O comes from a
// small row-dot kernel.  Two kernels keep every sum in a fixed order:
//
//   attn_bwd_dq_kernel  one item per (group, 128-query block); walks the key
//                       blocks at or below the diagonal:
//                         S = Q K^T, dP = dO V^T        (tensor memory)
//                         dS = P16 (dP - D) / sqrt(d)   (registers -> smem)
//                         dQ += dS K                    (tensor memory)
//   attn_bwd_kv_kernel  one item per (group, 128-key block); walks the query
//                       blocks at or above the diagonal:
//                         S^T = K Q^T, dP^T = V dO^T    (tensor memory)
//                         P^T, dS^T                     (registers -> smem)
//                         dV += P^T dO, dK += dS^T Q     (tensor memory)
//
// P16 is P rounded to the 16-bit type, as the matrix operand it is; dS uses
// the same rounded value.  Q, K, V and dO tiles are loaded once as 16-column
// chunks [128 rows][16] with 32-byte swizzle; the same tile serves as a
// K-major operand (reduction over head_dim) and, described differently, as
// an MN-major operand (reduction over the 128 rows).
//
// Warp roles (384 threads, one CTA per SM, persistent): warp 0 TMA; warp 1
// issues the S / dP MMAs, warp 10 the accumulating MMAs (dQ, or dV) and
// warp 11 those of dK, one thread each, so that the MMA streams run
// concurrently (warp 11 is idle in the dQ kernel); warps 2-9
// elementwise work: thread = (row, half of the 128 columns); warp w reads
// TMEM lane quarter w % 4.
#pragma once
#include <type_traits>

#include "common.cuh"

namespace gptl {

constexpr int kAttnBwdThreads = 384;   // 12 warps

struct AttnBwdParams {
  CUtensorMap map_c;     // C as [t*b][s][3h/t]; box {16, 128, 1}, 32B swizzle
  CUtensorMap map_do;    // dO as [t*b][s][h/t]; box {16, 128, 1}, 32B swizzle
  int s, d, hs, as;
  int groups, tiles;     // groups = t*b*heads per shard; tiles = ceil(s / 128)
  float scale_log2;      // log2(e) / sqrt(d)
  float scale;           // 1 / sqrt(d)
  uint32_t idesc_s;      // M 128, N 128, both K-major
  uint32_t idesc_acc;    // M 128, N d, A K-major, B MN-major
  const float *lse;      // [groups][s] base-2 log-sum-exp of the scaled scores
  const float *dvec;     // [groups][s] D = dO . O
  void *dc;              // [t*b*s][3h/t]: dQ, dK, dV written into their columns
  long long items;       // groups * tiles
  int q_off, k_off, v_off;
  int qdo_stages;        // dK/dV kernel: Q/dO ring depth (1..4)
  int kv_stages;         // dQ kernel: K/V ring depth (2..4)
  // bias-gradient partials (null: none): colsum[(bb * cs_rows + r) * cs_width
  // + i * 3h/t + column] = sum of the stored dQ/dK/dV values of shard i,
  // batch element bb, rows 32 r .. 32 r + 31 of the sequence
  float *colsum;
  int batch, cs_rows, cs_width;   // cs_rows = ceil(s / 32), cs_width = t * 3h/t
};

// The 32-row column sums of one warp's 16-column chunk (values as stored, 0
// for rows past the sequence) into the bias-gradient partials; zb = shard *
// batch + batch element, rgrp = the 32-row group of the sequence, col = the
// chunk's first column within the shard's 3h/t.
__device__ __forceinline__ void attn_colsum_chunk(const AttnBwdParams &p, const float (&v)[16],
                                                  int lane, int zb, int rgrp, int col) {
  const float sum = warp_colsum16(v, lane);
  if ((lane & 1) == 0 && rgrp < p.cs_rows)
    p.colsum[((long long)(zb % p.batch) * p.cs_rows + rgrp) * p.cs_width +
             (long long)(zb / p.batch) * (3 * p.hs) + col + ((lane >> 1) & 15)] = sum;
}

// A-operand tile [128 rows][128 cols] (16-bit), K-major, 128B swizzle: two
// 64-column atoms 16 KB apart.  Descriptor of k-step st (16 columns).
__device__ __forceinline__ uint64_t abwd_desc_a(uint32_t base, int st) {
  return make_smem_desc(base + (uint32_t)(st >> 2) * 16384u + (uint32_t)(st & 3) * 32u, 16u, 1024u, 2u);
}
// K-major chunk of 16 columns (reduction over head_dim), 32B swizzle.
__device__ __forceinline__ uint64_t abwd_desc_k16(uint32_t chunk) {
  return make_smem_desc(chunk, 16u, 256u, 6u);
}
// The same [d/16 chunks][128 rows][16] tile as an MN-major operand whose N is
// head_dim and whose reduction runs over the 128 rows: k-step st covers rows
// 16 st .. 16 st + 15 of every chunk.
__device__ __forceinline__ uint64_t abwd_desc_mn(uint32_t tile, int st) {
  return make_smem_desc(tile + (uint32_t)st * 512u, 4096u, 256u, 6u);
}
// Row `row`, 16-byte chunk c16 (0..15) of a [128][128] 16-bit A tile.
__device__ __forceinline__ uint32_t abwd_a_addr(uint32_t base, int row, int c16) {
  return base + (uint32_t)(c16 >> 3) * 16384u + (uint32_t)row * 128u +
         (uint32_t)(((c16 & 7) ^ (row & 7)) * 16);
}


// ============================================================ dQ kernel
template <typename T>
__global__ void __launch_bounds__(kAttnBwdThreads, 1)
    attn_bwd_dq_kernel(const __grid_constant__ AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int d = p.d;
  const uint32_t chunk = 128u * 32u;
  const uint32_t tb = (uint32_t)(d / 16) * chunk;             // one [128][d] tile
  const uint32_t ds_s = smem_u32(smem);                       // dS [128 q][128 keys]
  const uint32_t q_s = ds_s + 32768u, do_s = q_s + tb;
  const uint32_t kv_s = do_s + tb;                            // ring of K, V stages
  const uint32_t nkv = (uint32_t)p.kv_stages;                // K / V ring depth
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 32768u + 2u * tb + nkv * 2u * tb);
  const uint32_t qdo_full = smem_u32(&bars[0]), qdo_empty = smem_u32(&bars[1]);
  auto kv_full = [&](int i) { return smem_u32(&bars[2 + i]); };
  auto kv_empty = [&](int i) { return smem_u32(&bars[6 + i]); };
  const uint32_t sd_full = smem_u32(&bars[10]), sd_empty = smem_u32(&bars[11]);
  const uint32_t ds_full = smem_u32(&bars[12]), dq_done = smem_u32(&bars[13]);
  const uint32_t drain_bar = smem_u32(&bars[14]), drain_dq = smem_u32(&bars[15]);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 16);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(qdo_full, 1);
    mbar_init(qdo_empty, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(kv_full(i), 1);
      mbar_init(kv_empty(i), 1);
    }
    mbar_init(sd_full, 1);
    mbar_init(sd_empty, 8);
    mbar_init(ds_full, 8);
    mbar_init(dq_done, 1);
    mbar_init(drain_bar, 1);
    mbar_init(drain_dq, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.map_c);
    prefetch_tensormap(&p.map_do);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t t_s = tmem_base, t_dp = tmem_base + 128u, t_dq = tmem_base + 256u;

  // longest rows (last query blocks) first
  auto decode = [&](long long item, int &g, int &qb) {
    qb = p.tiles - 1 - (int)(item / p.groups);
    g = (int)(item % p.groups);
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t kv_it = 0, item_n = 0, issued = 0, parity_bits = 0;
      int q_parity = -1;
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x, ++item_n) {
        int g, qb;
        decode(item, g, qb);
        const int head = g % p.as, zb = g / p.as;
        if (!mbar_wait(qdo_empty, (item_n & 1u) ^ 1u, abort_flag)) goto tma_abort;
        mbar_arrive_expect_tx(qdo_full, 2u * tb);
        q_parity = (int)(item_n & 1u);
        for (int c = 0; c < d / 16; ++c) {
          tma_load_3d(q_s + (uint32_t)c * chunk, &p.map_c, p.q_off + head * d + c * 16, qb * 128, zb, qdo_full);
          tma_load_3d(do_s + (uint32_t)c * chunk, &p.map_do, head * d + c * 16, qb * 128, zb, qdo_full);
        }
        for (int j = 0; j <= qb; ++j, ++kv_it) {
          const int st = (int)(kv_it % nkv);
          const uint32_t ph = (kv_it / nkv) & 1u;
          if (!mbar_wait(kv_empty(st), ph ^ 1u, abort_flag)) goto tma_abort;
          mbar_arrive_expect_tx(kv_full(st), 2u * tb);
          const uint32_t k_s = kv_s + (uint32_t)st * 2u * tb, v_s = k_s + tb;
          for (int c = 0; c < d / 16; ++c) {
            tma_load_3d(k_s + (uint32_t)c * chunk, &p.map_c, p.k_off + head * d + c * 16, j * 128, zb, kv_full(st));
            tma_load_3d(v_s + (uint32_t)c * chunk, &p.map_c, p.v_off + head * d + c * 16, j * 128, zb, kv_full(st));
          }
          issued |= 1u << st;
          parity_bits = (parity_bits & ~(1u << st)) | (ph << st);
        }
      }
      goto tma_done;
    tma_abort:
      for (int s2 = 0; s2 < (int)nkv; ++s2)
        if (issued & (1u << s2)) mbar_wait_drain(kv_full(s2), (parity_bits >> s2) & 1u);
      if (q_parity >= 0) mbar_wait_drain(qdo_full, (uint32_t)q_parity);
    tma_done:;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------ MMA: S_j = Q K_j^T, dP_j = dO V_j^T
      uint32_t kv_it = 0, sd_it = 0, item_n = 0;
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x, ++item_n) {
        int g, qb;
        decode(item, g, qb);
        const int n = qb + 1;
        if (!mbar_wait(qdo_full, item_n & 1u, abort_flag)) goto mma_abort;
        tc_fence_after();
        for (int j = 0; j < n; ++j) {
          const uint32_t kj = kv_it + (uint32_t)j;
          if (!mbar_wait(kv_full((int)(kj % nkv)), (kj / nkv) & 1u, abort_flag)) goto mma_abort;
          if (!mbar_wait(sd_empty, (sd_it & 1u) ^ 1u, abort_flag)) goto mma_abort;
          ++sd_it;
          tc_fence_after();
          const uint32_t k_s = kv_s + (kj % nkv) * 2u * tb, v_s = k_s + tb;
          for (int c = 0; c < d / 16; ++c)
            tc_mma_f16(t_s, abwd_desc_k16(q_s + (uint32_t)c * chunk), abwd_desc_k16(k_s + (uint32_t)c * chunk),
                       p.idesc_s, c > 0 ? 1u : 0u);
          for (int c = 0; c < d / 16; ++c)
            tc_mma_f16(t_dp, abwd_desc_k16(do_s + (uint32_t)c * chunk), abwd_desc_k16(v_s + (uint32_t)c * chunk),
                       p.idesc_s, c > 0 ? 1u : 0u);
          tc_commit(sd_full);
        }
        tc_commit(qdo_empty);                // Q and dO are read by these MMAs only
        kv_it += (uint32_t)n;
      }
      goto mma_done;
    mma_abort:
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    mma_done:;
    }
  } else if (warp == 10) {
    if (lane == 0) {
      // ---------------------------------------------- MMA: dQ += dS_j K_j
      // A second issuing thread, alongside the S / dP MMAs.  dS_j exists only
      // after S_j and dP_j were read, so the K / V stage is free once this
      // block's dQ MMAs complete.
      uint32_t kv_it = 0, ds_it = 0;
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x) {
        int g, qb;
        decode(item, g, qb);
        const int n = qb + 1;
        for (int j = 0; j < n; ++j) {
          if (!mbar_wait(ds_full, ds_it & 1u, abort_flag)) goto dq_abort;
          ++ds_it;
          tc_fence_after();
          const uint32_t kj = kv_it + (uint32_t)j;
          const uint32_t k_s = kv_s + (kj % nkv) * 2u * tb;
          for (int st = 0; st < 8; ++st)   // dQ += dS K over the 128 keys
            tc_mma_f16(t_dq, abwd_desc_a(ds_s, st), abwd_desc_mn(k_s, st), p.idesc_acc,
                       (j > 0 || st > 0) ? 1u : 0u);
          tc_commit(dq_done);
          tc_commit(kv_empty((int)(kj % nkv)));
        }
        kv_it += (uint32_t)n;
      }
      goto dq_mma_done;
    dq_abort:
      tc_commit(drain_dq);
      mbar_wait_drain(drain_dq, 0);
    dq_mma_done:;
    }
  } else if (warp == 11) {
    // no role in this kernel (the block size is shared with the dK/dV kernel)
  } else {
    // ------------------------------------------- elementwise: one (row, half)
    const int q4 = warp & 3, half = (warp - 2) >> 2;
    const int row = q4 * 32 + lane;
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t col0 = (uint32_t)(half * 64);
    uint32_t sd_it = 0, dq_it = 0;
    for (long long item = blockIdx.x; item < p.items; item += gridDim.x) {
      int g, qb;
      decode(item, g, qb);
      const int n = qb + 1;
      const int qrow = qb * 128 + row;
      const bool valid_row = qrow < p.s;
      // P = exp2(S log2(e)/sqrt(d) - lse); dS = P16 (dP - D) / sqrt(d) as
      // P16 * (dP / sqrt(d) - D / sqrt(d))
      const float nl = valid_row ? -p.lse[(long long)g * p.s + qrow] : 0.f;
      const float nsdv = valid_row ? -p.scale * p.dvec[(long long)g * p.s + qrow] : 0.f;
      bool ok = true;
      for (int j = 0; j < n; ++j) {
        if (!mbar_wait(sd_full, sd_it & 1u, abort_flag)) { ok = false; break; }
        ++sd_it;
        tc_fence_after();
        const int key0 = j * 128 + (int)col0;
        // masking only where a key can be past the row or past the sequence
        const bool edge = (j == qb) || (j * 128 + 128 > p.s);
        // two passes over 32 of this thread's 64 columns each (bounded registers)
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t rs[2][16], rd[2][16];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tmem_ld16(t_s + lane_off + col0 + (uint32_t)((2 * hh + c) * 16), rs[c]);
            tmem_ld16(t_dp + lane_off + col0 + (uint32_t)((2 * hh + c) * 16), rd[c]);
          }
          tmem_wait_ld();
          if (hh == 1) {               // S / dP fully read: the MMAs may overwrite them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sd_empty);
          }
          uint32_t pk[16];                     // dS, packed pairs of 16-bit values
          auto block = [&](auto masked) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int e = 0; e < 16; e += 2) {
                float t0 = fmaf(__uint_as_float(rs[c][e]), p.scale_log2, nl);
                float t1 = fmaf(__uint_as_float(rs[c][e + 1]), p.scale_log2, nl);
                if (masked) {
                  const int key = key0 + (2 * hh + c) * 16 + e;
                  if (key > qrow || key >= p.s) t0 = -INFINITY;
                  if (key + 1 > qrow || key + 1 >= p.s) t1 = -INFINITY;
                }
                // P16: P rounded to the 16-bit operand type (exp2(-inf) = 0)
                const float2 pr = Cvt<T>::unpack2(Cvt<T>::pack2(ex2_approx(t0), ex2_approx(t1)));
                const float ds0 = pr.x * fmaf(__uint_as_float(rd[c][e]), p.scale, nsdv);
                const float ds1 = pr.y * fmaf(__uint_as_float(rd[c][e + 1]), p.scale, nsdv);
                pk[c * 8 + e / 2] = Cvt<T>::pack2(ds0, ds1);
              }
          };
          if (edge) block(std::true_type{});
          else block(std::false_type{});
          if (hh == 0 && j >= 1) {   // dQ += dS_{j-1} K_{j-1} done: the dS buffer is free
            if (!mbar_wait(dq_done, dq_it & 1u, abort_flag)) { ok = false; break; }
            ++dq_it;
          }
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16)
            st_shared_v4(abwd_a_addr(ds_s, row, half * 8 + hh * 4 + c16),
                         make_uint4(pk[4 * c16], pk[4 * c16 + 1], pk[4 * c16 + 2], pk[4 * c16 + 3]));
        }
        if (!ok) break;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ds_full);
      }
      if (!ok) break;
      if (!mbar_wait(dq_done, dq_it & 1u, abort_flag)) break;
      ++dq_it;
      tc_fence_after();
      // this thread stores half of the row's d columns
      const int head = g % p.as, zb = g / p.as;
      T *out = static_cast<T *>(p.dc) + ((long long)zb * p.s + qrow) * (3 * p.hs) + p.q_off + head * d;
      const int nch = d / 16;
      for (int c = half * ((nch + 1) / 2); c < (half ? nch : (nch + 1) / 2); ++c) {
        uint32_t o[16];
        tmem_ld16(t_dq + lane_off + (uint32_t)(c * 16), o);
        tmem_wait_ld();
        float cs[16];                  // the stored values, for the bias gradient
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[h2 * 8 + e]);
          const uint4 pk = pack8<T>(f);
          if (valid_row) reinterpret_cast<uint4 *>(out + c * 16)[h2] = pk;
          unpack8<T>(pk, f);
#pragma unroll
          for (int e = 0; e < 8; ++e) cs[h2 * 8 + e] = valid_row ? f[e] : 0.f;
        }
        if (p.colsum) attn_colsum_chunk(p, cs, lane, zb, qb * 4 + q4, p.q_off + head * d + c * 16);
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512u);
  }
}

// ========================================================== dK/dV kernel
template <typename T>
__global__ void __launch_bounds__(kAttnBwdThreads, 1)
    attn_bwd_kv_kernel(const __grid_constant__ AttnBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int d = p.d;
  const int nst = p.qdo_stages;
  const uint32_t chunk = 128u * 32u;
  const uint32_t tb = (uint32_t)(d / 16) * chunk;
  const uint32_t pt_s = smem_u32(smem);                       // P^T  [128 keys][128 q]
  const uint32_t dst_s = pt_s + 32768u;                       // dS^T [128 keys][128 q]
  const uint32_t k_s = dst_s + 32768u, v_s = k_s + tb;
  const uint32_t qdo_s = v_s + tb;                            // nst stages of Q, dO
  float *vecs = reinterpret_cast<float *>(smem + 65536u + 2u * tb + (uint32_t)nst * 2u * tb);
  // vecs: [2 buffers][lse 128, D 128]
  uint64_t *bars = reinterpret_cast<uint64_t *>(vecs + 512);
  const uint32_t kv_full = smem_u32(&bars[0]), kv_empty = smem_u32(&bars[1]);
  auto qdo_full = [&](int i) { return smem_u32(&bars[2 + i]); };
  auto qdo_empty = [&](int i) { return smem_u32(&bars[6 + i]); };
  const uint32_t sd_full = smem_u32(&bars[10]), sd_empty = smem_u32(&bars[11]);
  const uint32_t pds_full = smem_u32(&bars[12]), pds_free = smem_u32(&bars[13]);
  const uint32_t drain_bar = smem_u32(&bars[14]), drain_acc = smem_u32(&bars[17]);
  const uint32_t drain_acc2 = smem_u32(&bars[18]);
  auto vec_bar = [&](int i) { return smem_u32(&bars[15 + i]); };   // lse/D staged (256 arrivals)
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 19);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(vec_bar(0), 256);
    mbar_init(vec_bar(1), 256);
    mbar_init(kv_full, 1);
    mbar_init(kv_empty, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(qdo_full(i), 1);
      mbar_init(qdo_empty(i), 2);   // the dV and the dK issuer
    }
    mbar_init(sd_full, 1);
    mbar_init(sd_empty, 8);
    mbar_init(pds_full, 8);
    mbar_init(pds_free, 2);          // the dV and the dK issuer
    mbar_init(drain_bar, 1);
    mbar_init(drain_acc, 1);
    mbar_init(drain_acc2, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.map_c);
    prefetch_tensormap(&p.map_do);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t t_s = tmem_base, t_dp = tmem_base + 128u;
  const uint32_t t_dv = tmem_base + 256u, t_dk = tmem_base + 256u + (uint32_t)d;

  // longest columns (first key blocks) first
  auto decode = [&](long long item, int &g, int &kb) {
    kb = (int)(item / p.groups);
    g = (int)(item % p.groups);
  };

  if (warp == 0) {
    if (lane == 0) {
      uint32_t q_it = 0, item_n = 0, issued = 0, parity_bits = 0;
      int kv_parity = -1;
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x, ++item_n) {
        int g, kb;
        decode(item, g, kb);
        const int head = g % p.as, zb = g / p.as;
        if (!mbar_wait(kv_empty, (item_n & 1u) ^ 1u, abort_flag)) goto tma_abort;
        mbar_arrive_expect_tx(kv_full, 2u * tb);
        kv_parity = (int)(item_n & 1u);
        for (int c = 0; c < d / 16; ++c) {
          tma_load_3d(k_s + (uint32_t)c * chunk, &p.map_c, p.k_off + head * d + c * 16, kb * 128, zb, kv_full);
          tma_load_3d(v_s + (uint32_t)c * chunk, &p.map_c, p.v_off + head * d + c * 16, kb * 128, zb, kv_full);
        }
        for (int j = kb; j < p.tiles; ++j, ++q_it) {
          const int st = (int)(q_it % (uint32_t)nst);
          const uint32_t ph = (q_it / (uint32_t)nst) & 1u;
          if (!mbar_wait(qdo_empty(st), ph ^ 1u, abort_flag)) goto tma_abort;
          mbar_arrive_expect_tx(qdo_full(st), 2u * tb);
          const uint32_t q_s = qdo_s + (uint32_t)st * 2u * tb, do_s = q_s + tb;
          for (int c = 0; c < d / 16; ++c) {
            tma_load_3d(q_s + (uint32_t)c * chunk, &p.map_c, p.q_off + head * d + c * 16, j * 128, zb, qdo_full(st));
            tma_load_3d(do_s + (uint32_t)c * chunk, &p.map_do, head * d + c * 16, j * 128, zb, qdo_full(st));
          }
          issued |= 1u << st;
          parity_bits = (parity_bits & ~(1u << st)) | (ph << st);
        }
      }
      goto tma_done;
    tma_abort:
      for (int s2 = 0; s2 < nst; ++s2)
        if (issued & (1u << s2)) mbar_wait_drain(qdo_full(s2), (parity_bits >> s2) & 1u);
      if (kv_parity >= 0) mbar_wait_drain(kv_full, (uint32_t)kv_parity);
    tma_done:;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------- MMA: S^T = K Q_j^T, dP^T = V dO_j^T
      uint32_t q_it = 0, sd_it = 0, item_n = 0;
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x, ++item_n) {
        int g, kb;
        decode(item, g, kb);
        const int n = p.tiles - kb;
        if (!mbar_wait(kv_full, item_n & 1u, abort_flag)) goto mma_abort;
        tc_fence_after();
        for (int jj = 0; jj < n; ++jj) {
          const uint32_t qj = q_it + (uint32_t)jj;
          const int st = (int)(qj % (uint32_t)nst);
          if (!mbar_wait(qdo_full(st), (qj / (uint32_t)nst) & 1u, abort_flag)) goto mma_abort;
          if (!mbar_wait(sd_empty, (sd_it & 1u) ^ 1u, abort_flag)) goto mma_abort;
          ++sd_it;
          tc_fence_after();
          const uint32_t q_s = qdo_s + (uint32_t)st * 2u * tb, do_s = q_s + tb;
          for (int c = 0; c < d / 16; ++c)   // S^T = K Q^T
            tc_mma_f16(t_s, abwd_desc_k16(k_s + (uint32_t)c * chunk), abwd_desc_k16(q_s + (uint32_t)c * chunk),
                       p.idesc_s, c > 0 ? 1u : 0u);
          for (int c = 0; c < d / 16; ++c)   // dP^T = V dO^T
            tc_mma_f16(t_dp, abwd_desc_k16(v_s + (uint32_t)c * chunk), abwd_desc_k16(do_s + (uint32_t)c * chunk),
                       p.idesc_s, c > 0 ? 1u : 0u);
          tc_commit(sd_full);
        }
        tc_commit(kv_empty);                 // K and V are read by these MMAs only
        q_it += (uint32_t)n;
      }
      goto mma_done;
    mma_abort:
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    mma_done:;
    }
  } else if (warp == 10 || warp == 11) {
    if (lane == 0) {
      // -------------- MMA: dV += P_j^T dO_j (warp 10), dK += dS_j^T Q_j (warp 11)
      // Issuing threads of their own, alongside the S^T / dP^T MMAs.  P^T and
      // dS^T of block j exist only after its S^T / dP^T MMAs completed, so the
      // Q / dO stage is free once both of these streams complete block j.
      const bool is_dv = warp == 10;
      const uint32_t drain = is_dv ? drain_acc : drain_acc2;
      uint32_t q_it = 0, pds_it = 0;
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x) {
        int g, kb;
        decode(item, g, kb);
        const int n = p.tiles - kb;
        for (int jj = 0; jj < n; ++jj) {
          if (!mbar_wait(pds_full, pds_it & 1u, abort_flag)) goto acc_abort;
          ++pds_it;
          tc_fence_after();
          const uint32_t qj = q_it + (uint32_t)jj;
          const int st = (int)(qj % (uint32_t)nst);
          const uint32_t q_s = qdo_s + (uint32_t)st * 2u * tb, do_s = q_s + tb;
          for (int k2 = 0; k2 < 8; ++k2) {   // over the 128 queries
            const uint32_t acc = (jj > 0 || k2 > 0) ? 1u : 0u;
            if (is_dv) tc_mma_f16(t_dv, abwd_desc_a(pt_s, k2), abwd_desc_mn(do_s, k2), p.idesc_acc, acc);
            else tc_mma_f16(t_dk, abwd_desc_a(dst_s, k2), abwd_desc_mn(q_s, k2), p.idesc_acc, acc);
          }
          tc_commit(pds_free);
          tc_commit(qdo_empty(st));
        }
        q_it += (uint32_t)n;
      }
      goto acc_done;
    acc_abort:
      tc_commit(drain);
      mbar_wait_drain(drain, 0);
    acc_done:;
    }
  } else {
    // ------------------------------------------- elementwise: one (key row, half)
    const int q4 = warp & 3, half = (warp - 2) >> 2;
    const int row = q4 * 32 + lane;
    const int tid = threadIdx.x - 64;                 // 0..255
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t col0 = (uint32_t)(half * 64);
    uint32_t sd_it = 0, pds_it = 0, blk = 0;
    for (long long item = blockIdx.x; item < p.items; item += gridDim.x) {
      int g, kb;
      decode(item, g, kb);
      const int n = p.tiles - kb;
      const int key = kb * 128 + row;
      bool ok = true;
      // -lse and -D/sqrt(d) of one query block, for threads tid < 128
      auto vec_load = [&](int jq, float &a, float &b2) {
        const int q = jq * 128 + tid;
        a = q < p.s ? -p.lse[(long long)g * p.s + q] : 0.f;
        b2 = q < p.s ? -p.scale * p.dvec[(long long)g * p.s + q] : 0.f;
      };
      // Block j's vectors are staged in vecs[blk & 1] (double-buffered) and
      // published by vec_bar[blk & 1]: the first block's at the item start,
      // every later block's at the end of the block before it, from loads
      // issued at that block's start (their latency hides behind its work).
      // A thread passes block blk's barrier only after every thread has
      // finished block blk - 1, so the buffer rewritten at the end of block
      // blk (last read in block blk - 1) is free.
      float nl_next = 0.f, nd_next = 0.f;
      if (tid < 128) {
        vec_load(kb, nl_next, nd_next);
        vecs[(blk & 1u) * 256u + tid] = nl_next;
        vecs[(blk & 1u) * 256u + 128u + tid] = nd_next;
      }
      mbar_arrive(vec_bar((int)(blk & 1u)));
      for (int jj = 0; jj < n; ++jj, ++blk) {
        const int j = kb + jj;
        float *vb = vecs + (blk & 1u) * 256u;
        if (tid < 128 && jj + 1 < n) vec_load(j + 1, nl_next, nd_next);
        if (!mbar_wait(vec_bar((int)(blk & 1u)), (blk >> 1) & 1u, abort_flag)) { ok = false; break; }
        if (!mbar_wait(sd_full, sd_it & 1u, abort_flag)) { ok = false; break; }
        ++sd_it;
        tc_fence_after();
        // masking only where a query can be before the key or past the sequence
        const bool edge = (j == kb) || (j * 128 + 128 > p.s);
        const float4 *vb4 = reinterpret_cast<const float4 *>(vb);
        // two passes over 32 of this thread's 64 columns each, to bound the
        // registers held: load S^T and dP^T, form P16 and dS, store both
        for (int hh = 0; hh < 2; ++hh) {
          uint32_t rs[2][16], rd[2][16];
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tmem_ld16(t_s + lane_off + col0 + (uint32_t)((2 * hh + c) * 16), rs[c]);
            tmem_ld16(t_dp + lane_off + col0 + (uint32_t)((2 * hh + c) * 16), rd[c]);
          }
          tmem_wait_ld();
          if (hh == 1) {               // S^T / dP^T fully read: the MMAs may overwrite them
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(sd_empty);
          }
          uint32_t pp[16], pd[16];
          auto block = [&](auto masked) {
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
              for (int e = 0; e < 16; e += 4) {
                const int ql = (int)col0 + (2 * hh + c) * 16 + e;   // query within the block
                const float4 nl = vb4[ql / 4], nsdv = vb4[32 + ql / 4];
                float t[4] = {fmaf(__uint_as_float(rs[c][e]), p.scale_log2, nl.x),
                              fmaf(__uint_as_float(rs[c][e + 1]), p.scale_log2, nl.y),
                              fmaf(__uint_as_float(rs[c][e + 2]), p.scale_log2, nl.z),
                              fmaf(__uint_as_float(rs[c][e + 3]), p.scale_log2, nl.w)};
                if (masked) {
#pragma unroll
                  for (int u = 0; u < 4; ++u) {
                    const int q = j * 128 + ql + u;
                    if (q >= p.s || q < key) t[u] = -INFINITY;
                  }
                }
                // P16: P rounded to the 16-bit operand type (exp2(-inf) = 0)
                const uint32_t p01 = Cvt<T>::pack2(ex2_approx(t[0]), ex2_approx(t[1]));
                const uint32_t p23 = Cvt<T>::pack2(ex2_approx(t[2]), ex2_approx(t[3]));
                const float2 a = Cvt<T>::unpack2(p01), b = Cvt<T>::unpack2(p23);
                pp[c * 8 + e / 2] = p01;
                pp[c * 8 + e / 2 + 1] = p23;
                pd[c * 8 + e / 2] = Cvt<T>::pack2(a.x * fmaf(__uint_as_float(rd[c][e]), p.scale, nsdv.x),
                                                  a.y * fmaf(__uint_as_float(rd[c][e + 1]), p.scale, nsdv.y));
                pd[c * 8 + e / 2 + 1] =
                    Cvt<T>::pack2(b.x * fmaf(__uint_as_float(rd[c][e + 2]), p.scale, nsdv.z),
                                  b.y * fmaf(__uint_as_float(rd[c][e + 3]), p.scale, nsdv.w));
              }
          };
          if (edge) block(std::true_type{});
          else block(std::false_type{});
          if (hh == 0 && jj >= 1) {   // dV, dK of the previous block done: P^T and dS^T tiles free
            if (!mbar_wait(pds_free, pds_it & 1u, abort_flag)) { ok = false; break; }
            ++pds_it;
          }
#pragma unroll
          for (int c16 = 0; c16 < 4; ++c16) {
            const int col16 = half * 8 + hh * 4 + c16;
            st_shared_v4(abwd_a_addr(pt_s, row, col16),
                         make_uint4(pp[4 * c16], pp[4 * c16 + 1], pp[4 * c16 + 2], pp[4 * c16 + 3]));
            st_shared_v4(abwd_a_addr(dst_s, row, col16),
                         make_uint4(pd[4 * c16], pd[4 * c16 + 1], pd[4 * c16 + 2], pd[4 * c16 + 3]));
          }
        }
        if (!ok) break;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(pds_full);
        if (jj + 1 < n) {             // publish the next block's vectors
          if (tid < 128) {
            vecs[((blk + 1) & 1u) * 256u + tid] = nl_next;
            vecs[((blk + 1) & 1u) * 256u + 128u + tid] = nd_next;
          }
          mbar_arrive(vec_bar((int)((blk + 1) & 1u)));
        }
      }
      if (!ok) break;
      if (!mbar_wait(pds_free, pds_it & 1u, abort_flag)) break;
      ++pds_it;
      tc_fence_after();
      const int head = g % p.as, zb = g / p.as;
      const bool valid = key < p.s;
      T *rowp = static_cast<T *>(p.dc) + ((long long)zb * p.s + key) * (3 * p.hs) + head * d;
      const int nch = d / 16;
      for (int c = 0; c < nch; ++c) {
        // half 0 stores dV, half 1 stores dK
        uint32_t o[16];
        tmem_ld16((half ? t_dk : t_dv) + lane_off + (uint32_t)(c * 16), o);
        tmem_wait_ld();
        T *dst = rowp + (half ? p.k_off : p.v_off) + c * 16;
        const int col = (half ? p.k_off : p.v_off) + head * d + c * 16;   // within the shard's 3h/t
        float cs[16];                  // the stored values, for the bias gradient
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = __uint_as_float(o[h2 * 8 + e]);
          const uint4 pk = pack8<T>(f);
          if (valid) reinterpret_cast<uint4 *>(dst)[h2] = pk;
          unpack8<T>(pk, f);
#pragma unroll
          for (int e = 0; e < 8; ++e) cs[h2 * 8 + e] = valid ? f[e] : 0.f;
        }
        if (p.colsum) attn_colsum_chunk(p, cs, lane, zb, kb * 4 + q4, col);
      }
      tc_fence_before();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512u);
  }
}

}  // namespace gptl
