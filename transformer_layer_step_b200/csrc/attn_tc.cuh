// attn_tc.cuh — fused causal attention forward on tcgen05 (sm_100a).
//
// For every (shard, batch, head) and every 128-row block of queries, the
// kernel makes two passes over the 128-key blocks at or below the diagonal.
// Pass 1 computes S = Q K^T into tensor memory and reduces each row to its
// base-2 log-sum-exp lse = log2(sum_q 2^(S_pq log2(e)/sqrt(d))).  Pass 2
// computes S again, turns it into the normalised probabilities
// P = 2^(S log2(e)/sqrt(d) - lse), rounds them to the 16-bit type as the A
// operand of the next MMA (shared memory), and accumulates O += P V in tensor
// memory.  S and P never reach HBM.  This is the fused scale-mask-softmax of
// "Training GPT-2 with Megatron-LM" §6.2 (its output, the normalised P in
// 16 bits, is the operand of P V) carried one step further: the score matrix
// is consumed where it is produced.  Normalising before the rounding keeps
// the 16-bit operand exactly the one the unfused method multiplies; a single
// pass that rounds exp(S - running max) and divides by the row sum at the end
// would round different values.  The kernel writes O and lse, from which the
// backward recomputes P.
//
// Warp roles (640 threads, one CTA per SM, persistent over work items):
//   warp 0      TMA: Q once per item, then per key block K (pass 1) or K and
//               V (pass 2) into a ring of kv_stages (2..4) stages;
//   warp 1      one thread issues S_j = Q K_j^T into one of two S buffers;
//   warps 2-3   one thread each issues O += P_j V_j once P_j is ready, warp 2
//               over keys 0..63 of the block into O, warp 3 over keys 64..127
//               into O2 (added at the end): the MMA streams run concurrently;
//   warps 4-19  softmax: warp w reads TMEM lane quarter w % 4 (32 query rows,
//               one per thread) and quarter (w - 4) / 4 of the key block's
//               128 columns (32 columns), four warps per SM sub-partition to
//               hide the latency of their tensor-memory loads and exp2 chains.
//               Pass 1 keeps a running max and sum per quarter row; the four
//               quarters of a row meet once per item through shared memory to
//               form lse.  Pass 2 writes its 32 columns of P_j into one of two
//               shared-memory P buffers (so that P_j is formed while
//               P_{j-1} V_{j-1} runs).  At the end each warp stores its share
//               of O's columns.
// Tensor memory: S buffers at columns 0 and 128, O at column 256, O2 at 384.
// Shared memory: two P buffers [128 x 128] (two 128B-swizzled 64-column
// atoms each), Q as head_dim/16 chunks of [128 rows x 16] (32B swizzle), per
// stage K the same way and V as MN-major chunks of [64 keys x vw], then the
// barriers.  The quarter-row log-sum-exps are exchanged inside P buffer 0,
// which is idle between an item's passes: lane quarter q uses bytes
// [4096 q, +512) of its first atom, the rows that only q's warps write.
#pragma once
#include "common.cuh"

namespace gptl {

constexpr int kAttnThreads = 640;    // 20 warps: 4 roles + 16 softmax
constexpr int kAttnTile = 128;          // query rows per item, keys per block
constexpr int kAttnTailBytes = 256;     // barriers

struct AttnParams {
  CUtensorMap map_qk;   // C as [t*b][s][3h/t]; box {16, 128, 1}, 32B swizzle
  CUtensorMap map_v;    // same tensor; box {vw, 64, 1}
  int s, d, hs, as;     // sequence, head_dim, hidden per shard, heads per shard
  int groups;           // t * b * heads per shard
  int q_tiles;          // ceil(s / 128)
  int vw;               // V chunk width in elements (64, 32 or 16)
  float scale_log2;     // log2(e) / sqrt(head_dim)
  uint32_t idesc_s, idesc_pv;
  void *o;              // [t*b*s][h/t]
  float *lse;           // [groups][s]
  long long items;      // groups * q_tiles
  int q_off, k_off, v_off;   // column offsets of Q, K, V inside a shard's 3h/t columns
  int kv_stages;             // depth of the K / V ring (2..4)
};

// K-major operand chunk of 16 columns, 32B swizzle: rows of 32 B, 8-row
// groups 256 B apart.
__device__ __forceinline__ uint64_t attn_desc_k16(uint32_t addr) {
  return make_smem_desc(addr, 16u, 256u, 6u);
}

// log2(2^a + 2^b) for the two halves of a row (either may be -inf); the
// same value whichever half computes it.
__device__ __forceinline__ float lse_merge(float a, float b) {
  const float mx = fmaxf(a, b);
  if (mx == -INFINITY) return -INFINITY;
  return mx + log2f(ex2_approx(a - mx) + ex2_approx(b - mx));
}

template <typename T>
__global__ void __launch_bounds__(kAttnThreads, 1) attn_fwd_kernel(const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  const int d = p.d;
  const uint32_t chunk_bytes = 128u * 32u;                   // one 16-column chunk, 128 rows
  const uint32_t q_bytes = (uint32_t)(d / 16) * chunk_bytes;  // = 128 * d * 2
  const uint32_t kv_bytes = 2u * q_bytes;                     // K and V of one stage
  const uint32_t p_s = smem_u32(smem);                        // P: two 32 KB buffers
  const uint32_t q_s = p_s + 65536u;
  const uint32_t kv_s = q_s + q_bytes;
  const uint32_t nkv = (uint32_t)p.kv_stages;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 65536u + q_bytes + nkv * kv_bytes);
  // bars: q_full q_empty kv_full[4] kv_empty[4] s_full[2] s_empty[2] p_full[2] pv_done[2]
  //       stat_full[4] stat_read[4] drain drain_pv[2]
  const uint32_t q_full = smem_u32(&bars[0]), q_empty = smem_u32(&bars[1]);
  auto kv_full = [&](int i) { return smem_u32(&bars[2 + i]); };
  auto kv_empty = [&](int i) { return smem_u32(&bars[6 + i]); };
  auto s_full = [&](int i) { return smem_u32(&bars[10 + i]); };
  auto s_empty = [&](int i) { return smem_u32(&bars[12 + i]); };
  // P_j (pass 2) lives in buffer j % 2 (j counted over all of the CTA's
  // pass-2 blocks): p_full[b] publishes it, pv_done[b] reports its P V
  // products complete
  auto p_full = [&](int b) { return smem_u32(&bars[14 + b]); };
  auto pv_done = [&](int b) { return smem_u32(&bars[16 + b]); };
  // the four softmax warps of lane quarter q exchange their quarter-row lse
  auto stat_full = [&](int q) { return smem_u32(&bars[18 + q]); };
  auto stat_read = [&](int q) { return smem_u32(&bars[22 + q]); };
  const uint32_t drain_bar = smem_u32(&bars[26]);
  auto drain_pv = [&](int h) { return smem_u32(&bars[27 + h]); };
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 29);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(kv_full(i), 1);
      mbar_init(kv_empty(i), 2);   // pass 2: both P V issuers; pass 1: two commits of the S issuer
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(s_full(i), 1);
      mbar_init(s_empty(i), 16);   // the sixteen softmax warps
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(p_full(b), 16);
      mbar_init(pv_done(b), 2);    // both halves of P_j V_j
    }
    for (int q = 0; q < 4; ++q) {
      mbar_init(stat_full(q), 128);  // every thread of the quarter's four warps
      mbar_init(stat_read(q), 128);
    }
    mbar_init(drain_bar, 1);
    mbar_init(drain_pv(0), 1);
    mbar_init(drain_pv(1), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&p.map_qk);
    prefetch_tensormap(&p.map_v);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_o = tmem_base + 256u;    // O over keys 0..63 of each block
  const uint32_t tmem_o2 = tmem_base + 384u;   // O over keys 64..127 (added at the end)

  // work item -> (group, query block): the longest rows (last query blocks) first
  auto decode = [&](long long item, int &g, int &qt) {
    qt = p.q_tiles - 1 - (int)(item / p.groups);
    g = (int)(item % p.groups);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA
      uint32_t kv_it = 0, item_n = 0;
      uint32_t issued = 0, parity_bits = 0;   // stages with loads in flight, for a clean abort
      int q_parity = -1;                      // parity of the last Q load issued
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x, ++item_n) {
        int g, qt;
        decode(item, g, qt);
        const int head = g % p.as, zb = g / p.as;
        const int n = qt + 1;
        if (!mbar_wait(q_empty, (item_n & 1u) ^ 1u, abort_flag)) goto tma_abort;
        mbar_arrive_expect_tx(q_full, q_bytes);
        q_parity = (int)(item_n & 1u);
        for (int c = 0; c < d / 16; ++c)
          tma_load_3d(q_s + (uint32_t)c * chunk_bytes, &p.map_qk, p.q_off + head * d + c * 16,
                      qt * kAttnTile, zb, q_full);
        for (int it = 0; it < 2 * n; ++it, ++kv_it) {
          const int j = it < n ? it : it - n;
          const bool with_v = it >= n;            // pass 2
          const int st = (int)(kv_it % nkv);
          const uint32_t ph = (kv_it / nkv) & 1u;
          if (!mbar_wait(kv_empty(st), ph ^ 1u, abort_flag)) goto tma_abort;
          mbar_arrive_expect_tx(kv_full(st), with_v ? kv_bytes : q_bytes);
          const uint32_t k_s = kv_s + (uint32_t)st * kv_bytes, v_s = k_s + q_bytes;
          for (int c = 0; c < d / 16; ++c)
            tma_load_3d(k_s + (uint32_t)c * chunk_bytes, &p.map_qk, p.k_off + head * d + c * 16,
                        j * kAttnTile, zb, kv_full(st));
          if (with_v) {
            const int nvc = d / p.vw;
            for (int kb = 0; kb < 2; ++kb)
              for (int c = 0; c < nvc; ++c)
                tma_load_3d(v_s + (uint32_t)((kb * nvc + c) * 64 * p.vw * 2), &p.map_v,
                            p.v_off + head * d + c * p.vw, j * kAttnTile + kb * 64, zb, kv_full(st));
          }
          issued |= 1u << st;
          parity_bits = (parity_bits & ~(1u << st)) | (ph << st);
        }
      }
      goto tma_done;
    tma_abort:
      for (int s2 = 0; s2 < (int)nkv; ++s2)
        if (issued & (1u << s2)) mbar_wait_drain(kv_full(s2), (parity_bits >> s2) & 1u);
      if (q_parity >= 0) mbar_wait_drain(q_full, (uint32_t)q_parity);
    tma_done:;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------ MMA: S_j = Q K_j^T
      uint32_t kv_it = 0, s_it = 0, item_n = 0;
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x, ++item_n) {
        int g, qt;
        decode(item, g, qt);
        const int n = qt + 1;
        if (!mbar_wait(q_full, item_n & 1u, abort_flag)) goto mma_abort;
        tc_fence_after();
        for (int it = 0; it < 2 * n; ++it) {
          const uint32_t kj = kv_it + (uint32_t)it;
          if (!mbar_wait(kv_full((int)(kj % nkv)), (kj / nkv) & 1u, abort_flag)) goto mma_abort;
          const int sb = (int)(s_it & 1u);
          if (!mbar_wait(s_empty(sb), ((s_it >> 1) & 1u) ^ 1u, abort_flag)) goto mma_abort;
          tc_fence_after();
          const uint32_t k_s = kv_s + (kj % nkv) * kv_bytes;
          for (int c = 0; c < d / 16; ++c)
            tc_mma_f16(tmem_base + (uint32_t)(sb * 128), attn_desc_k16(q_s + (uint32_t)c * chunk_bytes),
                       attn_desc_k16(k_s + (uint32_t)c * chunk_bytes), p.idesc_s, c > 0 ? 1u : 0u);
          tc_commit(s_full(sb));
          if (it < n) {                      // pass 1: the stage held K only, now read
            tc_commit(kv_empty((int)(kj % nkv)));
            tc_commit(kv_empty((int)(kj % nkv)));
          }
          ++s_it;
        }
        tc_commit(q_empty);                  // Q is read by these MMAs only
        kv_it += (uint32_t)(2 * n);
      }
      goto mma_done;
    mma_abort:
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    mma_done:;
    }
  } else if (warp == 2 || warp == 3) {
    if (lane == 0) {
      // ------------------------------------------- MMA: O += P_j V_j
      // Second and third issuing threads: their MMAs run alongside the S
      // MMAs.  P_j exists only after S_j was read, so K_j is no longer in use
      // when the stage is released here.
      const int h = warp - 2;
      uint32_t kv_it = 0, pb = 0;              // pb: the CTA's pass-2 block counter (P buffer pb % 2)
      for (long long item = blockIdx.x; item < p.items; item += gridDim.x) {
        int g, qt;
        decode(item, g, qt);
        const int n = qt + 1;
        for (int j = 0; j < n; ++j, ++pb) {
          const int buf = (int)(pb & 1u);
          if (!mbar_wait(p_full(buf), (pb >> 1) & 1u, abort_flag)) goto pv_abort;
          tc_fence_after();
          const uint32_t pbuf = p_s + (uint32_t)buf * 32768u;
          const uint32_t pj = kv_it + (uint32_t)(n + j);
          const uint32_t v_s = kv_s + (pj % nkv) * kv_bytes + q_bytes;
          const uint32_t row_b = (uint32_t)p.vw * 2u;
          const uint32_t kb_bytes = (uint32_t)(d / p.vw) * 64u * row_b;
          const uint32_t vsw = p.vw == 64 ? 2u : (p.vw == 32 ? 4u : 6u);
          // issuer 0: keys 0..63 of the block into O, issuer 1: keys 64..127 into O2
          const uint32_t acc_t = h == 0 ? tmem_o : tmem_o2;
          for (int st = 0; st < 4; ++st) {
            const uint64_t adesc =
                make_smem_desc(pbuf + (uint32_t)h * 16384u + (uint32_t)st * 32u, 16u, 1024u, 2u);
            const uint64_t bdesc = make_smem_desc(v_s + (uint32_t)h * kb_bytes + (uint32_t)st * 16u * row_b,
                                                  64u * row_b, 8u * row_b, vsw);
            tc_mma_f16(acc_t, adesc, bdesc, p.idesc_pv, (j > 0 || st > 0) ? 1u : 0u);
          }
          tc_commit(pv_done(buf));
          tc_commit(kv_empty((int)(pj % nkv)));
        }
        kv_it += (uint32_t)(2 * n);
      }
      goto pv_done;
    pv_abort:
      tc_commit(drain_pv(h));
      mbar_wait_drain(drain_pv(h), 0);
    pv_done:;
    }
  } else {
    // -------------------------------------------------- softmax and epilogue
    const int q4 = warp & 3;                 // TMEM lane quarter of this warp
    const int qc = (warp - 4) >> 2;          // which 32 of the block's 128 keys
    const int row = q4 * 32 + lane;          // query row within the block
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    // the quarter-row lse exchange of lane quarter q4 (inside P buffer 0)
    float *xlse = reinterpret_cast<float *>(smem + q4 * 4096);
    uint32_t s_it = 0, pb = 0, item_n = 0;   // pb: the CTA's pass-2 block counter
    // wait until the P V products of pass-2 block k are done; only ever
    // called for the latest block that used P buffer k % 2
    auto wait_pv = [&](uint32_t k) { return mbar_wait(pv_done((int)(k & 1u)), (k >> 1) & 1u, abort_flag); };
    // S_j, columns [qc * 32, +32) of S buffer s_it % 2, masked past the
    // diagonal and the sequence end; releases the S buffer
    auto read_s = [&](int j, int qrow, uint32_t (&r)[2][16]) -> bool {
      const int sb = (int)(s_it & 1u);
      if (!mbar_wait(s_full(sb), (s_it >> 1) & 1u, abort_flag)) return false;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c)
        tmem_ld16(tmem_base + lane_off + (uint32_t)(sb * 128 + qc * 32 + c * 16), r[c]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty(sb));
      ++s_it;
      const int key0 = j * kAttnTile + qc * 32;
      if (j * kAttnTile + kAttnTile - 1 >= qrow - row || key0 + 32 > p.s) {
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int key = key0 + c * 16 + e;
            if (key > qrow || key >= p.s) r[c][e] = __float_as_uint(-INFINITY);
          }
      }
      return true;
    };
    for (long long item = blockIdx.x; item < p.items; item += gridDim.x, ++item_n) {
      int g, qt;
      decode(item, g, qt);
      const int n = qt + 1;
      const int qrow = qt * kAttnTile + row;
      bool ok = true;
      // ---- pass 1: running max m and sum l of 2^(S c) over this quarter row
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        uint32_t r[2][16];
        if (!read_s(j, qrow, r)) { ok = false; break; }
        float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 16; e += 4)
#pragma unroll
            for (int k = 0; k < 4; ++k) mx[k] = fmaxf(mx[k], __uint_as_float(r[c][e + k]));
        const float m_new = fmaxf(m, fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale_log2);
        if (m_new == -INFINITY) continue;      // every key so far masked
        const float nm = -m_new;
        float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 2; ++c)
#pragma unroll
          for (int e = 0; e < 16; e += 4)
#pragma unroll
            for (int k = 0; k < 4; ++k)
              sm[k] += ex2_approx(fmaf(__uint_as_float(r[c][e + k]), p.scale_log2, nm));
        l = l * (m_new == m ? 1.0f : ex2_approx(m - m_new)) + ((sm[0] + sm[1]) + (sm[2] + sm[3]));
        m = m_new;
      }
      if (!ok) break;
      // ---- the row's lse from its four quarters (shared memory, once per
      // item; P buffer 0 is idle here: the previous item's P V products all
      // completed before its O was stored)
      const float lse_q = l > 0.f ? m + log2f(l) : -INFINITY;
      xlse[qc * 32 + lane] = lse_q;
      mbar_arrive(stat_full(q4));
      if (!mbar_wait(stat_full(q4), item_n & 1u, abort_flag)) break;
      const float l0 = xlse[lane], l1 = xlse[32 + lane], l2 = xlse[64 + lane], l3 = xlse[96 + lane];
      mbar_arrive(stat_read(q4));
      // every warp of the quarter forms the same value, in the same order
      const float lse = lse_merge(lse_merge(l0, l1), lse_merge(l2, l3));
      const float nl = lse == -INFINITY ? 0.f : -lse;
      // the exchange slots are read by all four warps before P overwrites them
      if (!mbar_wait(stat_read(q4), item_n & 1u, abort_flag)) break;
      // ---- pass 2: P = 2^(S c - lse) in 16 bits, the A operand of P V
      for (int j = 0; j < n; ++j, ++pb) {
        uint32_t r[2][16];
        if (!read_s(j, qrow, r)) { ok = false; break; }
        // P buffer pb % 2 is free once block pb-2's P V products are done (an
        // earlier item's blocks are all done: its end waited for its last)
        if (j >= 2 && !wait_pv(pb - 2)) { ok = false; break; }
        // this quarter's 32 columns: 16-byte chunks 4 (qc % 2) .. + 3 of atom
        // qc / 2 of the 128B-swizzled K-major A tile; chunk c8 of row `row`
        // goes to slot c8 ^ (row % 8)
        const uint32_t pbuf = p_s + (pb & 1u) * 32768u + (uint32_t)(qc >> 1) * 16384u + (uint32_t)row * 128u;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            f[e] = ex2_approx(fmaf(__uint_as_float(r[i >> 1][(i & 1) * 8 + e]), p.scale_log2, nl));
          const int c8 = (qc & 1) * 4 + i;
          st_shared_v4(pbuf + (uint32_t)((c8 ^ (row & 7)) * 16), pack8<T>(f));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(p_full((int)(pb & 1u)));
      }
      if (!ok) break;
      // ---- epilogue: wait for the last P V, store this warp's share of O
      // (16-column chunks [qc nc / 4, (qc + 1) nc / 4)) and the lse
      if (!wait_pv(pb - 1)) break;
      tc_fence_after();
      const int head = g % p.as, zb = g / p.as;
      T *orow = static_cast<T *>(p.o) + ((long long)zb * p.s + qrow) * p.hs + head * d;
      const int nc = d / 16;
      for (int c = (qc * nc) / 4; c < ((qc + 1) * nc) / 4; ++c) {
        uint32_t o[16], o2[16];
        tmem_ld16(tmem_o + lane_off + (uint32_t)(c * 16), o);
        tmem_ld16(tmem_o2 + lane_off + (uint32_t)(c * 16), o2);
        tmem_wait_ld();
        if (qrow < p.s) {
          float f[8];
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              f[e] = __uint_as_float(o[h2 * 8 + e]) + __uint_as_float(o2[h2 * 8 + e]);
            reinterpret_cast<uint4 *>(orow + c * 16)[h2] = pack8<T>(f);
          }
        }
      }
      if (qc == 0 && qrow < p.s) p.lse[(long long)g * p.s + qrow] = lse;
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
