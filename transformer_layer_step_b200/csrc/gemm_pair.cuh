// gemm_pair.cuh — the tcgen05 GEMM on CTA pairs (cta_group::2), sm_100a.
//
// The same contraction and epilogues as gemm_tc_kernel, with each output
// tile of 256 x BN computed by a cluster of two CTAs on two SMs.  The leader
// CTA (rank 0) issues tcgen05.mma.cta_group::2 with M = 256: rows 0..127 of
// the tile accumulate in the leader's tensor memory, rows 128..255 in the
// peer's, and the B tile (BN rows of N) is read half from each CTA's shared
// memory.  So each SM stages 128 rows of A and BN/2 rows of B per k-block:
// the operand bytes per FLOP of a 256 x BN tile, at half the shared memory
// per stage, which leaves room for a deep ring (up to 6 stages of 32 KB) and
// for two accumulators of BN columns in each SM's tensor memory: the
// epilogue of one tile overlaps the MMAs of the next.
//
// Roles (384 threads per CTA, one CTA per SM, persistent over tiles; both
// CTAs of a pair walk the same tile sequence):
//   warp 0     TMA producer in both CTAs: its own A rows and B half into its
//              own ring; the copies complete on the LEADER's full barrier
//              (cp.async.bulk.tensor ... .cta_group::2, no multicast), whose
//              expected byte count the leader's producer sets for both;
//   warp 1     allocates the pair's tensor memory (tcgen05.alloc.cta_group::2
//              in both CTAs); in the leader, one thread issues the MMAs and
//              commits each stage's release to the empty barriers of both
//              CTAs, and each finished accumulator to both tfull barriers
//              (tcgen05.commit ... .multicast::cluster);
//   warps 4-11 epilogue in both CTAs: drain this CTA's 128 rows of the
//              accumulator (as gemm_tc_kernel's epilogue warps), then arrive
//              on the leader's tempty barrier (16 arrivals free it).
// Every wait is bounded as in gemm_tc_kernel.  No load uses multicast: each
// CTA reads its operands from this GPU's memory itself.
#pragma once
#include "gemm_tc.cuh"

namespace gptl {

constexpr int kPairThreads = 384;
constexpr int kPairMaxStages = 6;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// shared::cluster address of the variable at shared address `addr` in CTA `rank`
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(addr), "r"(rank));
  return d;
}

// every thread of both CTAs
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// arrive on an mbarrier in another CTA of the cluster (shared::cluster address)
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(20u)
      : "memory");
  return ok != 0;
}

// mbar_wait for a barrier that other CTAs of the cluster arrive on
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int *abort) {
  const unsigned long long t0 = globaltimer();
#pragma unroll 1
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 1024; ++i)
      if (mbar_try_wait_cluster(bar, parity)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > kWaitTimeoutNs) {
      set_device_error(kErrTimeout);
      *abort = 1;
      return false;
    }
  }
}

// 3-D tiled TMA load into this CTA's shared memory, completing on an
// mbarrier of either CTA of the pair (bar: shared::cluster address)
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *map, int x, int y,
                                                 int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void load_operand_pair(const CUtensorMap *map, const OperandRule &r,
                                                  uint32_t dst, int rows, int g, int ks, int mn0,
                                                  int k0, uint32_t bar) {
  const int x0 = (g % r.x_mod) * r.x_mul + r.x_off;
  const int gc = g / r.g_div + (r.k_shard ? ks : 0);
  if (!r.mn_major) {
    tma_load_3d_pair(dst, map, x0 + k0, mn0, gc, bar);
  } else {
    const int chunks = rows / r.w;
    for (int c = 0; c < chunks; ++c)
      tma_load_3d_pair(dst + (uint32_t)(c * kBK * r.w * 2), map, x0 + mn0 + c * r.w, k0, gc, bar);
  }
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D (M = 256 over the pair) (+)= A * B, kind::f16
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                                uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the mbarrier at this shared offset in every CTA of `mask`
// when all earlier tcgen05 ops of this thread have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

template <typename T>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    gemm_pair_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const uint32_t rank = cluster_ctarank();
  const int b_rows = p.bn / 2;                     // this CTA's rows of the B tile
  const int a_bytes = kBM * kBK * 2;
  const int stage_bytes = a_bytes + b_rows * kBK * 2;
  const int S = p.stages;
  const uint32_t staging_s = smem_u32(smem + S * stage_bytes);   // 1024-aligned
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + S * stage_bytes + kStagingBytes);
  // bars: full[S] empty[S] tfull[2] tempty[2] drain
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * S + 5);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t tiles_s = smem_u32(smem);
  auto full_bar = [&](int s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](int s) { return smem_u32(&bars[S + s]); };
  auto tfull_bar = [&](int a) { return smem_u32(&bars[2 * S + a]); };
  auto tempty_bar = [&](int a) { return smem_u32(&bars[2 * S + 2 + a]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * S + 4]);
  auto stage_addr = [&](int s) { return tiles_s + (uint32_t)(s * stage_bytes); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full_bar(s), 1);                   // the leader's expect_tx arrival
      mbar_init(empty_bar(s), 1);                  // one multicast commit per use
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 2 * kEpiWarps);     // both CTAs' epilogue warps
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.map_a);
    prefetch_tensormap(&p.map_b);
    prefetch_tensormap(&p.map_o);
    if (p.act == kActGelu) prefetch_tensormap(&p.map_o2);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), (uint32_t)p.tmem_cols);
    tmem_relinquish_pair();
  }
  // both CTAs' barriers initialised and tensor memory allocated before any
  // copy or MMA of the pair touches them
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer (both CTAs)
      int stage = 0;
      uint32_t phase = 0, issued = 0, parity = 0;
      for (long long idx = pair; idx < p.total_tiles; idx += npairs) {
        const TileInfo ti = tile_info(p, idx);
        for (int ks = 0; ks < p.k_shards; ++ks)
          for (int kb = ti.kb_begin; kb < ti.kb_end; ++kb) {
            if (!mbar_wait(empty_bar(stage), phase ^ 1, abort_flag)) goto producer_abort;
            const uint32_t fb = full_bar(stage);
            if (rank == 0) mbar_arrive_expect_tx(fb, (uint32_t)(2 * stage_bytes));
            const uint32_t fb_leader = mapa_shared(fb, 0);
            const uint32_t sa = stage_addr(stage);
            load_operand_pair(&p.map_a, p.ra, sa, kBM, ti.g, ks, ti.m0 + (int)rank * kBM, kb * kBK,
                              fb_leader);
            load_operand_pair(&p.map_b, p.rb, sa + a_bytes, b_rows, ti.g, ks,
                              ti.n0 + (int)rank * b_rows, kb * kBK, fb_leader);
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
      // the leader sees every copy of the pair land on its full barriers
      if (rank == 0)
        for (int s = 0; s < S; ++s)
          if (issued & (1u << s)) mbar_wait_drain(full_bar(s), (parity >> s) & 1u);
    producer_done:;
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------ MMA issuer (leader)
      int stage = 0;
      uint32_t phase = 0, acc_phase[2] = {0u, 0u};
      int t = 0;
      for (long long idx = pair; idx < p.total_tiles; idx += npairs, ++t) {
        const TileInfo ti = tile_info(p, idx);
        const int acc = t & 1;
        if (!mbar_wait_cluster(tempty_bar(acc), acc_phase[acc] ^ 1, abort_flag)) goto mma_abort;
        acc_phase[acc] ^= 1;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * p.bn_alloc);
        int it = 0;
        for (int ks = 0; ks < p.k_shards; ++ks)
          for (int kb = ti.kb_begin; kb < ti.kb_end; ++kb) {
            if (!mbar_wait(full_bar(stage), phase, abort_flag)) goto mma_abort;
            tc_fence_after();
            const uint32_t sa = stage_addr(stage);
            const uint32_t sb = sa + (uint32_t)a_bytes;
            const int nsteps = min(kBK, p.K - kb * kBK) / 16;
            for (int s = 0; s < nsteps; ++s)
              tc_mma_f16_pair(d_tmem, operand_desc(p.ra, sa, s), operand_desc(p.rb, sb, s), p.idesc,
                              (it > 0 || s > 0) ? 1u : 0u);
            tc_commit_pair(empty_bar(stage), (uint16_t)3);
            ++it;
            if (++stage == S) {
              stage = 0;
              phase ^= 1;
            }
          }
        tc_commit_pair(tfull_bar(acc), (uint16_t)3);
      }
      goto mma_done;
    mma_abort:
      // wait for the MMAs already issued before tensor memory is released
      tc_commit_pair(drain_bar, (uint16_t)1);
      mbar_wait_drain(drain_bar, 0);
    mma_done:;
    }
  } else if (warp >= 4) {
    // -------------------------------------------------- epilogue warps (both CTAs)
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - 4) >> 2;        // which half of the tile's columns
    const bool wide = p.out_f32 != 0;        // fp32: one chunk per box
    const bool gelu = !wide && p.act == kActGelu;
    const uint32_t my_boxes = staging_s + (uint32_t)((warp - 4) * 2 * kStageBoxBytes);
    const uint32_t tempty_leader[2] = {mapa_shared(tempty_bar(0), 0), mapa_shared(tempty_bar(1), 0)};
    int box_i = 0;
    bool bad = false;
    uint32_t acc_phase[2] = {0u, 0u};
    int t = 0;
    for (long long idx = pair; idx < p.total_tiles; idx += npairs, ++t) {
      const TileInfo ti = tile_info(p, idx);
      const int acc = t & 1;
      if (!mbar_wait(tfull_bar(acc), acc_phase[acc], abort_flag)) break;
      acc_phase[acc] ^= 1;
      tc_fence_after();
      const int row0 = ti.m0 + (int)rank * kBM + q * 32;
      const EpiRow er = epilogue_row<T>(p, ti.g, row0 + lane);
      const uint32_t t_row = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * p.bn_alloc);
      int oz, ow;
      if (p.o_flat) { oz = ti.g; ow = 0; }
      else { oz = ti.g % p.o_mod; ow = ti.g / p.o_mod; }
      const int nchunk = p.bn / 16;
      const int csplit = 2 * ((nchunk + 3) / 4);
      const int c0 = half ? csplit : 0;
      int c1 = half ? nchunk : csplit;
      const int valid = (p.N - ti.n0 + 15) / 16;
      if (c1 > valid) c1 = valid;
      uint32_t ra[16], rb[16];
      EpiIn ia, ib;
      auto ld = [&](int c, uint32_t (&r)[16]) { tmem_ld16(t_row + (uint32_t)(c * 16), r); };
      auto process = [&](int c, const uint32_t (&r)[16], const EpiIn &in) {
        const int slot = wide ? 0 : ((c - c0) & 1);
        const bool first = slot == 0, last = wide || slot == 1 || c + 1 == c1;
        const uint32_t buf = my_boxes + (uint32_t)((gelu ? 0 : (box_i & 1)) * kStageBoxBytes);
        if (first) {
          if (lane == 0) {
            if (gelu) bulk_wait_read<0>();
            else bulk_wait_read<1>();
          }
          __syncwarp();
        }
        epilogue_chunk<T>(p, er, r, in, buf, my_boxes + kStageBoxBytes, lane, slot, bad);
        if (last) {
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int x = ti.n0 + (c - slot) * 16;
            tma_store_4d(&p.map_o, buf, x, row0, oz, ow);
            if (gelu) tma_store_4d(&p.map_o2, my_boxes + kStageBoxBytes, x, row0, oz, ow);
            bulk_commit();
          }
          ++box_i;
        }
      };
      if (c0 < c1) {
        ld(c0, ra);
        epilogue_load<T>(p, er, ti.n0 + c0 * 16, ia);
        tmem_wait_ld();
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
        const bool has_a = c + 2 < c1;
        if (has_a) {
          ld(c + 2, ra);
          epilogue_load<T>(p, er, ti.n0 + (c + 2) * 16, ia);
        }
        process(c + 1, rb, ib);
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(tempty_leader[acc]);
    }
    if (p.nonfinite && __any_sync(0xffffffffu, bad) && lane == 0) atomicOr(p.nonfinite, 1);
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  // both CTAs done with every MMA, copy and tensor-memory read of the pair
  tc_fence_before();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, (uint32_t)p.tmem_cols);
  }
}

}  // namespace gptl
