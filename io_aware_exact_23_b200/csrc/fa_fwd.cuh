// fa_fwd.cuh -- fused exact-attention forward kernel for sm_100a.
//
// One CTA computes O and LSE for a pair of 128-row query tiles of one head:
// the "tile inputs / compute locally / online normalisation / write compact
// output" steps of the FlashAttention summary ("Architecture, step by step"),
// with the online softmax of the review's "Tiling" section.  The N x N scores
// live only in tensor memory (TMEM), one 128 x 128 tile at a time.
//
// Roles (320 threads):
//   warps 0-3  softmax for query tile 0 (thread t owns row t, TMEM lane t)
//   warps 4-7  softmax for query tile 1
//   warp  8    TMA producer: Q0, Q1 once, then K_j / V_j through a smem ring
//   warp  9    MMA issuer (one thread): S_k = Q_k K_j^T and O_k += P_k V_j
//
// TMEM columns (512 allocated): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D).  P_k (bf16, two per column) overwrites the first 64
// columns of S_k once the softmax threads hold S_k in registers.
//
// Online softmax, in the log2 domain with c = scale*log2(e):
//   m' = max(m, c*rowmax(S));  P = 2^(c*S - m');  l = 2^(m-m') l + rowsum(P);
//   O = 2^(m-m') O + P V.
// O is divided by the row sum of P as rounded to bf16 (the weights the MMA
// actually applied), LSE uses the fp32 row sum.
// The running max is only moved when it grows by more than 8 (a factor 256):
// O and l are both kept relative to the same stale max, which is exact, and
// P <= 256 cannot overflow fp32 or bf16.  Most tiles then skip the O rescale.
#pragma once

#include "ptx.cuh"

namespace fa {

struct FwdParams {
  float *lse;        // [BH, N] fp32 (natural log)
  uint16_t *o_lo;    // optional [BH, N, D] bf16: bf16(O_fp32 - O), or nullptr
  int *status;       // device status block
  int seq;           // launch sequence number (for the status block)
  int N;
  int BH;
  int n_qpairs;      // ceil(N / 256)
  float scale_log2;  // scale * log2(e)
};

template <int D>
struct FwdCfg {
  static constexpr int kTileBytes = 128 * D * 2;      // one 128 x D bf16 tile
  static constexpr int kStages = (D == 128) ? 4 : 6;  // K/V ring depth
  static constexpr int kBoxes = D / 64;               // 64-column TMA boxes per tile
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kBarOff = kKVOff + kStages * kTileBytes;
  static constexpr int kSmemBytes = kBarOff + 512;
  static constexpr int kThreads = 320;
};

enum FwdTag : int {
  kTagQ = 1, kTagKvFull = 2, kTagKvEmpty = 3, kTagSFull = 4, kTagPFull = 5, kTagPvDone = 6, kTagEpi = 7
};

// Position of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled
// tile: TMA's SWIZZLE_128B pattern XORs the chunk index with row % 8.
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}

template <int D, bool CAUSAL>
__global__ void __launch_bounds__(320, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const FwdParams p) {
  using C = FwdCfg<D>;
  extern __shared__ __align__(1024) uint8_t smem[];

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
  uint64_t *bar_q = bars + 0;                        // [2]
  uint64_t *bar_kv_full = bars + 2;                  // [kStages]
  uint64_t *bar_kv_empty = bars + 2 + C::kStages;    // [kStages]
  uint64_t *bar_s_full = bars + 2 + 2 * C::kStages;  // [2]
  uint64_t *bar_p_full = bar_s_full + 2;             // [2]
  uint64_t *bar_pv_done = bar_p_full + 2;            // [2]
  uint64_t *bar_epi = bar_pv_done + 2;               // [2]
  uint64_t *bar_drain = bar_epi + 2;                 // [1]
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_drain + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: longest-first over query-tile pairs (matters when causal).
  const int bh = blockIdx.x % p.BH;
  const int u = p.n_qpairs - 1 - static_cast<int>(blockIdx.x / p.BH);
  const int n_kv_all = (p.N + 127) / 128;
  int n_kv0, n_kv1;  // KV tiles seen by query tile 0 / 1
  if (CAUSAL) {
    n_kv0 = min(2 * u + 1, n_kv_all);
    n_kv1 = min(2 * u + 2, n_kv_all);
  } else {
    n_kv0 = n_kv_all;
    n_kv1 = n_kv_all;
  }
  const int n_kv = n_kv1;  // n_kv1 >= n_kv0

  const WaitCtx ctx{p.status, abort_flag, kKernelFwd, p.seq};

  if (threadIdx.x == 0) {
    // The swizzle arithmetic and the UMMA descriptors assume a 1024-byte
    // aligned shared-memory window.
    *abort_flag = 0;
    if ((smem_u32(smem) & 1023u) != 0) record_failure(ctx, kStatusInternal, 0);
    mbar_init(&bar_q[0], 1);
    mbar_init(&bar_q[1], 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bar_kv_full[s], 1);
      mbar_init(&bar_kv_empty[s], 1);
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bar_s_full[k], 1);
      mbar_init(&bar_p_full[k], 128);
      mbar_init(&bar_pv_done[k], 1);
      mbar_init(&bar_epi[k], 128);
    }
    mbar_init(bar_drain, 1);
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  uint8_t *sQ = smem + C::kQOff;
  uint8_t *sKV = smem + C::kKVOff;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      tma_prefetch_desc(&tmO);
      mbar_arrive_expect_tx(&bar_q[0], C::kTileBytes);
      for (int b = 0; b < C::kBoxes; ++b)
        tma_load_3d(&tmQ, &bar_q[0], sQ + b * 16384, b * 64, (2 * u) * 128, bh);
      int idx = 0;
      bool ok = true;
      for (int j = 0; j < n_kv && ok; ++j) {
        for (int t = 0; t < 2 && ok; ++t) {
          const int s = idx % C::kStages, n = idx / C::kStages;
          if (n > 0 && !mbar_wait(ctx, &bar_kv_empty[s], (n - 1) & 1, kTagKvEmpty)) { ok = false; break; }
          uint8_t *dst = sKV + s * C::kTileBytes;
          mbar_arrive_expect_tx(&bar_kv_full[s], C::kTileBytes);
          for (int b = 0; b < C::kBoxes; ++b)
            tma_load_3d(t == 0 ? &tmK : &tmV, &bar_kv_full[s], dst + b * 16384, b * 64, j * 128, bh);
          ++idx;
          if (j == 0 && t == 0) {
            mbar_arrive_expect_tx(&bar_q[1], C::kTileBytes);
            for (int b = 0; b < C::kBoxes; ++b)
              tma_load_3d(&tmQ, &bar_q[1], sQ + C::kTileBytes + b * 16384, b * 64, (2 * u + 1) * 128, bh);
          }
        }
      }
      if (!ok) {
        // Drain the copies still in flight before the CTA can exit.
        mbar_drain(&bar_q[0], 0);
        if (idx > 0) mbar_drain(&bar_q[1], 0);
        for (int s = 0; s < C::kStages && s < idx; ++s) {
          const int last = s + ((idx - 1 - s) / C::kStages) * C::kStages;
          mbar_drain(&bar_kv_full[s], (last / C::kStages) & 1);
        }
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && !*abort_flag) {
      constexpr uint32_t idesc_qk = make_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = make_idesc_bf16(128, D, 0, 1);
      const uint32_t q_addr[2] = {smem_u32(sQ), smem_u32(sQ + C::kTileBytes)};
      const uint32_t kv_addr = smem_u32(sKV);
      const uint32_t tS[2] = {tmem, tmem + 128};
      const uint32_t tO[2] = {tmem + 256, tmem + 256 + D};
      bool ok = mbar_wait(ctx, &bar_q[0], 0, kTagQ);
      for (int j = 0; j < n_kv && ok; ++j) {
        const int iK = 2 * j, iV = 2 * j + 1;
        const int sK = iK % C::kStages, sV = iV % C::kStages;
        ok = mbar_wait(ctx, &bar_kv_full[sK], (iK / C::kStages) & 1, kTagKvFull);
        if (!ok) break;
        tc_fence_after();
        const uint32_t k_addr = kv_addr + sK * C::kTileBytes;
        for (int k = 0; k < 2 && ok; ++k) {
          if (k == 0 && j >= n_kv0) continue;
          if (k == 1 && j == 0) ok = mbar_wait(ctx, &bar_q[1], 0, kTagQ);
          // S_k is free once PV_k of the previous tile has consumed P_k.
          if (ok && j > 0) ok = mbar_wait(ctx, &bar_pv_done[k], (j - 1) & 1, kTagPvDone);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
            mma_ss(tS[k], make_sdesc(q_addr[k] + off, 16, 1024), make_sdesc(k_addr + off, 16, 1024), idesc_qk,
                   ks > 0);
          }
          mma_commit(&bar_s_full[k]);
        }
        if (!ok) break;
        mma_commit(&bar_kv_empty[sK]);
        ok = mbar_wait(ctx, &bar_kv_full[sV], (iV / C::kStages) & 1, kTagKvFull);
        if (!ok) break;
        tc_fence_after();
        const uint32_t v_addr = kv_addr + sV * C::kTileBytes;
        for (int k = 0; k < 2 && ok; ++k) {
          if (k == 0 && j >= n_kv0) continue;
          ok = mbar_wait(ctx, &bar_p_full[k], j & 1, kTagPFull);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            mma_ts(tO[k], tS[k] + ks * 8, make_sdesc(v_addr + ks * 2048, 16384, 1024), idesc_pv,
                   (j > 0 || ks > 0) ? 1u : 0u);
          }
          mma_commit(&bar_pv_done[k]);
        }
        if (!ok) break;
        mma_commit(&bar_kv_empty[sV]);
      }
      if (!ok) {
        // Let every MMA already issued finish before TMEM is released.
        mma_commit(bar_drain);
        mbar_drain(bar_drain, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int k = warp >> 2;  // query tile handled by this warpgroup
    const int r = (warp & 3) * 32 + lane;  // row within the tile == TMEM lane
    const int qt = 2 * u + k;              // query tile index
    const int n_k = (k == 0) ? n_kv0 : n_kv1;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lane_off + 128 * k;
    const uint32_t tO = tmem + lane_off + 256 + k * D;
    const float c = p.scale_log2;
    float m = -INFINITY, l = 0.f, lr = 0.f;  // running max, row sum, rounded row sum
    bool ok = !*abort_flag;
    for (int j = 0; j < n_k && ok; ++j) {
      ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_s_full[k], j & 1, kTagSFull));
      if (!ok) break;
      tc_fence_after();
      uint32_t s[128];
      tmem_ld32(tS + 0, s + 0);
      tmem_ld32(tS + 32, s + 32);
      tmem_ld32(tS + 64, s + 64);
      tmem_ld32(tS + 96, s + 96);
      tmem_wait_ld();
      // Keys j*128 + col are valid when col < nvalid (tail of N, causal diagonal).
      int nvalid = min(128, p.N - j * 128);
      if (CAUSAL && j == qt) nvalid = min(nvalid, r + 1);
      if (nvalid < 128) {
#pragma unroll
        for (int cc = 0; cc < 128; ++cc)
          if (cc >= nvalid) s[cc] = __float_as_uint(-INFINITY);
      }
      float mx = __uint_as_float(s[0]);
#pragma unroll
      for (int cc = 1; cc < 128; ++cc) mx = fmaxf(mx, __uint_as_float(s[cc]));
      const float m_cand = mx * c;
      float alpha = 1.f;
      bool rescale = false;
      if (m_cand > m + 8.f) {  // also taken on the first tile (m = -inf)
        alpha = ex2(m - m_cand);
        rescale = (j > 0);
        m = m_cand;
      }
      const float neg = (m == -INFINITY) ? 0.f : -m;
      // Two row sums: of P in fp32 (for the LSE) and of P as rounded to bf16,
      // i.e. exactly the weights the PV MMA multiplies V with (for O's
      // normaliser, so that O is a convex combination of the rows of V).
      float sum0 = 0.f, sum1 = 0.f, rsum0 = 0.f, rsum1 = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int cc = 0; cc < 64; ++cc) {
        const float a = ex2(fmaf(__uint_as_float(s[2 * cc]), c, neg));
        const float b = ex2(fmaf(__uint_as_float(s[2 * cc + 1]), c, neg));
        sum0 += a;
        sum1 += b;
        pk[cc] = pack_bf16(a, b);
        rsum0 += __uint_as_float(pk[cc] << 16);
        rsum1 += __uint_as_float(pk[cc] & 0xFFFF0000u);
      }
      l = l * alpha + (sum0 + sum1);
      lr = lr * alpha + (rsum0 + rsum1);
      if (__any_sync(0xffffffffu, rescale)) {
        // O_k still holds the previous tile's PV: wait for it, then rescale.
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_pv_done[k], (j - 1) & 1, kTagPvDone));
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < D / 32; ++ch) {
          uint32_t o[32];
          tmem_ld32(tO + ch * 32, o);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
          tmem_st32(tO + ch * 32, o);
        }
      }
      tmem_st32(tS + 0, pk + 0);
      tmem_st32(tS + 32, pk + 32);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p_full[k]);
    }
    // ---------------------------------------------------------- epilogue
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_pv_done[k], (n_k - 1) & 1, kTagPvDone));
    if (ok) {
      tc_fence_after();
      const float inv_l = 1.f / lr;
      uint8_t *stage = sQ + k * C::kTileBytes;  // Q_k is dead: all its MMAs completed
      const uint32_t stage_addr = smem_u32(stage);
#pragma unroll
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(tO + ch * 32, o);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int t = 0; t < 16; ++t)
          w[t] = pack_bf16(__uint_as_float(o[2 * t]) * inv_l, __uint_as_float(o[2 * t + 1]) * inv_l);
        if (p.o_lo != nullptr && qt * 128 + r < p.N) {
          // What rounding O to bf16 dropped, itself rounded to bf16: O ~ o + o_lo
          // to about 16 significant bits (used by the backward's D = rowsum(dO o O)).
          uint32_t lo[16];
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            const float a = __uint_as_float(o[2 * t]) * inv_l, b = __uint_as_float(o[2 * t + 1]) * inv_l;
            lo[t] = pack_bf16(a - __uint_as_float(w[t] << 16), b - __uint_as_float(w[t] & 0xFFFF0000u));
          }
          uint4 *dst = reinterpret_cast<uint4 *>(p.o_lo + (static_cast<size_t>(bh) * p.N + qt * 128 + r) * D +
                                                 ch * 32);
#pragma unroll
          for (int t = 0; t < 4; ++t) dst[t] = make_uint4(lo[4 * t], lo[4 * t + 1], lo[4 * t + 2], lo[4 * t + 3]);
        }
        const int box = ch >> 1;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const int chunk = (ch & 1) * 4 + t;
          st_shared_v4(stage_addr + box * 16384 + sw128_offset(r, chunk), w[4 * t], w[4 * t + 1], w[4 * t + 2],
                       w[4 * t + 3]);
        }
      }
      const int grow = qt * 128 + r;
      if (grow < p.N) p.lse[static_cast<size_t>(bh) * p.N + grow] = (m + log2f(l)) * 0.69314718055994531f;
      // Make the generic-proxy smem writes visible to TMA, then one thread of
      // the warpgroup stores the tile once all 128 rows have arrived.
      fence_proxy_async_smem();
      mbar_arrive(&bar_epi[k]);
      if (r == 0 && mbar_wait(ctx, &bar_epi[k], 0, kTagEpi) && qt * 128 < p.N) {
        for (int b = 0; b < C::kBoxes; ++b) tma_store_3d(&tmO, stage + b * 16384, b * 64, qt * 128, bh);
        bulk_commit();
        bulk_wait_read<0>();
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 9) tmem_dealloc(tmem, 512);
}

}  // namespace fa
