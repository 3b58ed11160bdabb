// fa_fwd.cuh -- fused exact-attention forward kernel for sm_100a.
//
// One CTA computes O and LSE for a pair of 128-row query tiles of one head:
// the "tile inputs / compute locally / online normalisation / write compact
// output" steps of the FlashAttention summary ("Architecture, step by step"),
// with the online softmax of the review's "Tiling" section.  The N x N scores
// live only on chip, one 128 x 128 tile at a time: the fp32 S
// and the bf16 P in tensor memory (TMEM).
//
// Roles (352 threads):
//   warps 0-7  softmax.  Warp w owns rows 32*(w%4)..+31 (its TMEM lane
//              quarter) and the column half h = w/4 of every S tile.  All eight
//              warps work on tile 0 of KV step j, then on tile 1, then on tile 0
//              of step j+1 ...: while they run one tile's softmax, the tensor
//              pipe runs the other tile's PV and next S.  The two warps that
//              share rows exchange their half-row maxima through smem.
//   warp  8    TMA producer: Q0, Q1 once, then K / V tiles through a smem ring.
//   warp  9    MMA issuer for tile 0 (one thread); warp 10 for tile 1.  Two
//              independent issuers let the pipe take whichever tile is ready.
// A K/V ring stage is released when both issuers' MMAs that read it completed.
//
// TMEM columns (512 allocated): S0 [0,128), S1 [128,256), O0 [256,256+D),
// O1 [256+D, 256+2D).  The bf16 P (two per column) of column half h is written
// over S columns [64h, 64h+32) -- inside the half its warp has already read --
// and is the A operand of the PV MMA straight from TMEM.  The next S of a tile
// overwrites those columns; its issuer puts it in the pipe right behind that
// tile's PV (one issuing thread: the MMAs execute in order), without waiting.
//
// Online softmax, in the log2 domain with c = scale*log2(e):
//   m' = max(m, c*rowmax(S));  P = 2^(c*S - m');  l = 2^(m-m') l + rowsum(P);
//   O = 2^(m-m') O + P V.
// O is divided by the row sum of P as rounded to bf16 (the weights the MMA
// actually applied), LSE uses the fp32 row sum.
// The running max is only moved when it grows by more than 8 (a factor 256):
// O and l are both kept relative to the same stale max, which is exact, and
// P <= 256 cannot overflow fp32 or bf16.  Most tiles then skip the O rescale.
// After the first KV step P is computed against the running max before the
// row max of the new tile is known (the half maxima travel through smem in the
// meantime); only a row whose max grew by more than 8 recomputes its P.
// Every exponential runs on the MUFU unit (one per 4d FLOPs; at d = 128 its
// rate equals the tensor rate).  Moving a share of them to the FMA pipe as a
// polynomial was measured slower: FP32-pipe pressure from the softmax warps
// delays the MMA issue more than the MUFU queue does.
#pragma once

#include "dropout.cuh"
#include "ptx.cuh"

namespace fa {

struct FwdParams {
  uint16_t *o;       // [BH, N, D] bf16
  float *lse;        // [BH, N] fp32 (natural log)
  uint16_t *o_lo;    // optional [BH, N, D] bf16: bf16(O_fp32 - O), or nullptr
  int *status;       // device status block
  int seq;           // launch sequence number (for the status block)
  int N;
  int BH;
  int n_qpairs;      // ceil(N / 256)
  float scale_log2;  // scale * log2(e)
  DropoutParams drop;  // read only by the DROPOUT instantiations
  // FP8 instantiations only: per-head descale factors [BH] of the e4m3 Q, K, V
  // (the inputs are code * descale).
  const float *descale_q, *descale_k, *descale_v;
};

// FP8: Q, K, V as e4m3 (one byte per element); the output O stays bf16.
template <int D, bool FP8 = false>
struct FwdCfg {
  static_assert(!FP8 || D == 128, "the e4m3 forward takes d = 128 (one 128-byte swizzle row per tile row)");
  static constexpr int kElemBytes = FP8 ? 1 : 2;
  static constexpr int kTileBytes = 128 * D * kElemBytes;  // one 128 x D input tile
  static constexpr int kBoxCols = 128 / kElemBytes;        // input elements per 128-byte TMA box row
  static constexpr int kBoxes = kTileBytes / 16384;        // 128-row TMA boxes (16 KB) per input tile
  static constexpr int kStages = (FP8 || D == 64) ? 8 : 4;  // K/V ring depth
  // The epilogue stages each softmax warp's 32 rows of O and o_lo (bf16, D/2
  // columns each) in the idle ring.
  static_assert(kStages * kTileBytes >= 8 * 2 * 32 * D, "epilogue staging");
  static constexpr int kQOff = 0;
  static constexpr int kKVOff = 2 * kTileBytes;
  static constexpr int kXOff = kKVOff + kStages * kTileBytes;  // half-row maxima [2 tiles][2 halves][128]
  static constexpr int kLOff = kXOff + 2048;                   // half-row sums [2 tiles][2 halves][2][128]
  static constexpr int kBarOff = kLOff + 4096;
  // mbarriers: q[2], kv_full/kv_empty[kStages], s_full/p_full/pv_done/drain
  // [2] each (one per query tile), the max and sum exchanges [2][4] (one per
  // tile and warp pair); then the TMEM address slot and the abort flag.
  static constexpr int kNumBars = 2 + 2 * kStages + 24;
  static constexpr int kSmemBytes = kBarOff + kNumBars * 8 + 16;
  static constexpr int kThreads = 352;
  static constexpr int kSoftmaxThreads = 256;
  static constexpr int kProducerWarp = 8;
  static constexpr int kIssuerWarp = 9;  // 9: tile 0 (and TMEM owner), 10: tile 1
  static_assert(kSmemBytes <= 232448, "shared memory budget");
};

enum FwdTag : int {
  kTagQ = 1, kTagKvFull = 2, kTagKvEmpty = 3, kTagSFull = 4, kTagPFull = 5, kTagPvDone = 6, kTagEpi = 7,
  kTagXmax = 8, kTagLsum = 9
};

// Load order of the K/V ring: K tiles run one KV step ahead of V tiles
// (K0, K1, V0, K2, V1, ..., K_{n-1}, V_{n-2}, V_{n-1}), because S of step j+1
// is issued while P of step j is still being computed.  Ring slot of each load:
__device__ __forceinline__ int kv_idx_k(int j) { return j == 0 ? 0 : 2 * j - 1; }
__device__ __forceinline__ int kv_idx_v(int j, int n) { return (j + 1 < n) ? 2 * j + 2 : 2 * j + 1; }

// Position of 16-byte chunk `chunk` (0..7) of row `row` in a 128-byte-swizzled
// tile: TMA's SWIZZLE_128B pattern XORs the chunk index with row % 8.
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk) {
  return static_cast<uint32_t>(row * 128 + ((chunk ^ (row & 7)) << 4));
}


// FP8: e4m3 Q, K, V with per-head descale factors (kind::f8f6f4 MMAs, K = 32
// per instruction); P is rounded to e4m3 for the PV product, four per TMEM
// column, and O is divided by the fp32 row sum of the unrounded P.
template <int D, bool CAUSAL, bool DROPOUT = false, bool FP8 = false>
__global__ void __launch_bounds__(352, 1)
    fa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  static_assert(!(FP8 && DROPOUT), "no dropout in the e4m3 forward");
  using C = FwdCfg<D, FP8>;
  extern __shared__ __align__(1024) uint8_t smem[];
  if (threadIdx.x == 0) FA_TRACE(1);

  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::kBarOff);
  uint64_t *bar_q = bars + 0;                        // [2]
  uint64_t *bar_kv_full = bars + 2;                  // [kStages]
  uint64_t *bar_kv_empty = bars + 2 + C::kStages;    // [kStages]
  uint64_t *bar_s_full = bars + 2 + 2 * C::kStages;  // [2] S_k in TMEM
  uint64_t *bar_p_full = bar_s_full + 2;             // [2] P_k in TMEM (and O_k rescaled)
  uint64_t *bar_pv_done = bar_p_full + 2;            // [2] PV_k completed
  uint64_t *bar_drain = bar_pv_done + 2;             // [2] abort path: the issuer's MMAs completed
  uint64_t *bar_x = bar_drain + 2;                   // [2][4] half-row max exchange, per warp pair
  uint64_t *bar_l = bar_x + 8;                       // [2][4] half-row sum exchange, per warp pair
  static_assert(2 + 2 * C::kStages + 24 == C::kNumBars, "barrier count");
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_l + 8);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Work unit: heads in chunks of 8 (their K/V stay resident in L2 while the
  // chunk runs); inside a chunk, longest query-tile pairs first (causal).
  int bh, u;
  {
    constexpr int kChunk = 8;
    const int per_chunk = kChunk * p.n_qpairs;
    const int ch = static_cast<int>(blockIdx.x) / per_chunk, rem = static_cast<int>(blockIdx.x) % per_chunk;
    const int g = min(kChunk, p.BH - ch * kChunk);
    u = p.n_qpairs - 1 - rem / g;
    bh = ch * kChunk + rem % g;
  }
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
      mbar_init(&bar_kv_empty[s], 2);  // one arrival per MMA issuer
    }
    for (int k = 0; k < 2; ++k) {
      mbar_init(&bar_s_full[k], 1);
      mbar_init(&bar_p_full[k], C::kSoftmaxThreads);
      mbar_init(&bar_pv_done[k], 1);
      for (int q = 0; q < 4; ++q) {
        // Warps q and q+4 share rows 32q..32q+31 (and an SM sub-partition).
        mbar_init(&bar_x[k * 4 + q], 64);
        mbar_init(&bar_l[k * 4 + q], 64);
      }
      mbar_init(&bar_drain[k], 1);
    }
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == C::kIssuerWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) FA_TRACE(0);

  uint8_t *sQ = smem + C::kQOff;
  uint8_t *sKV = smem + C::kKVOff;

  if (warp == C::kProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && !*abort_flag) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      mbar_arrive_expect_tx(&bar_q[0], C::kTileBytes);
      for (int b = 0; b < C::kBoxes; ++b)
        tma_load_3d(&tmQ, &bar_q[0], sQ + b * 16384, b * C::kBoxCols, (2 * u) * 128, bh);
      int idx = 0;
      bool ok = true;
      for (; idx < 2 * n_kv && ok; ++idx) {
        // Which tile is load number idx in the K-ahead order.
        const bool is_k = (idx == 0) || ((idx & 1) && (idx + 1) / 2 < n_kv);
        const int j = (idx == 0) ? 0 : (is_k ? (idx + 1) / 2 : (idx == 2 * n_kv - 1 ? n_kv - 1 : idx / 2 - 1));
        const int s = idx % C::kStages, n = idx / C::kStages;
        if (n > 0 && !mbar_wait(ctx, &bar_kv_empty[s], (n - 1) & 1, kTagKvEmpty)) { ok = false; break; }
        uint8_t *dst = sKV + s * C::kTileBytes;
        mbar_arrive_expect_tx(&bar_kv_full[s], C::kTileBytes);
        for (int b = 0; b < C::kBoxes; ++b)
          tma_load_3d(is_k ? &tmK : &tmV, &bar_kv_full[s], dst + b * 16384, b * C::kBoxCols, j * 128, bh);
        if (idx == 0) {
          mbar_arrive_expect_tx(&bar_q[1], C::kTileBytes);
          for (int b = 0; b < C::kBoxes; ++b)
            tma_load_3d(&tmQ, &bar_q[1], sQ + C::kTileBytes + b * 16384, b * C::kBoxCols, (2 * u + 1) * 128, bh);
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
  } else if (warp == C::kIssuerWarp || warp == C::kIssuerWarp + 1) {
    // ------------------------------------------------------------ MMA issuers
    const int k = warp - C::kIssuerWarp;  // query tile owned by this issuer
    if (lane == 0 && !*abort_flag) {
      constexpr uint32_t idesc_qk = FP8 ? make_idesc_e4m3(128, 128, 0, 0) : make_idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = FP8 ? make_idesc_e4m3(128, D, 0, 1) : make_idesc_bf16(128, D, 0, 1);
      // Base descriptors: Q_k (K-major), ring stage 0 as K (K-major) and as V (MN-major).
      const uint64_t q_desc = make_sdesc(smem_u32(sQ + k * C::kTileBytes), 16, 1024);
      const uint64_t k_desc0 = make_sdesc(smem_u32(sKV), 16, 1024);
      const uint64_t v_desc0 = make_sdesc(smem_u32(sKV), 16384, 1024);
      const uint32_t tS = tmem + 128 * k;
      const uint32_t tO = tmem + 256 + k * D;
      const int n_k = (k == 0) ? n_kv0 : n_kv1;
      bool ok = mbar_wait(ctx, &bar_q[k], 0, kTagQ);
      for (int j = 0; j < n_kv && ok; ++j) {
        const int iK = kv_idx_k(j), sK = iK % C::kStages;
        const int iV = kv_idx_v(j, n_kv), sV = iV % C::kStages;
        // Arrivals on kv_empty must follow the matching kv_full phase, so even
        // a tile that skips K_j / V_j (causal tile 0 past its diagonal) waits.
        ok = mbar_wait(ctx, &bar_kv_full[sK], (iK / C::kStages) & 1, kTagKvFull);
        if (!ok) break;
        if (j >= n_k) {
          mbar_arrive(&bar_kv_empty[sK]);
          ok = mbar_wait(ctx, &bar_kv_full[sV], (iV / C::kStages) & 1, kTagKvFull);
          if (ok) mbar_arrive(&bar_kv_empty[sV]);
          continue;
        }
        // S_k aliases P_k, which the previous PV_k reads.  Both MMAs come from
        // this thread and the tensor pipe runs them in issue order, so S_k is
        // issued right behind PV_k without waiting for it to complete.
        const uint64_t k_desc = sdesc_add(k_desc0, sK * C::kTileBytes);
        // One MMA per 32-byte K slice of the 128-byte swizzled rows (16 bf16 or 32 e4m3).
#pragma unroll
        for (int ks = 0; ks < D * C::kElemBytes / 32; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          if constexpr (FP8)
            mma_ss_f8(tS, sdesc_add(q_desc, off), sdesc_add(k_desc, off), idesc_qk, ks > 0);
          else
            mma_ss(tS, sdesc_add(q_desc, off), sdesc_add(k_desc, off), idesc_qk, ks > 0);
        }
        mma_commit(&bar_s_full[k]);
        mma_commit(&bar_kv_empty[sK]);
        FA_TRACE(16 + k * 256 + 4 * j + 0);
        ok = mbar_wait(ctx, &bar_kv_full[sV], (iV / C::kStages) & 1, kTagKvFull);
        if (ok) ok = mbar_wait(ctx, &bar_p_full[k], j & 1, kTagPFull);
        if (!ok) break;
        tc_fence_after();
        FA_TRACE(16 + k * 256 + 4 * j + 2);
        const uint64_t v_desc = sdesc_add(v_desc0, sV * C::kTileBytes);
        // K steps over the 128 keys: 16 (bf16) or 32 (e4m3) keys, 8 TMEM columns of P
        // and 16 or 32 rows of V each; P of keys 64h.. starts at column 64h.
        if constexpr (FP8) {
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_ts_f8(tO, tS + ks * 8 + (ks >= 2 ? 48 : 0), sdesc_add(v_desc, ks * 4096), idesc_pv,
                      (j > 0 || ks > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ts(tO, tS + ks * 8 + (ks >= 4 ? 32 : 0), sdesc_add(v_desc, ks * 2048), idesc_pv,
                   (j > 0 || ks > 0) ? 1u : 0u);
        }
        mma_commit(&bar_pv_done[k]);
        mma_commit(&bar_kv_empty[sV]);
        FA_TRACE(16 + k * 256 + 4 * j + 1);
      }
      if (!ok) {
        // Let every MMA this thread issued finish before TMEM is released.
        mma_commit(&bar_drain[k]);
        mbar_drain(&bar_drain[k], 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int h = warp >> 2;                 // column half of every S tile
    const int rq = warp & 3;                 // TMEM lane quarter
    const int r = rq * 32 + lane;            // row within the tile == TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(rq * 32) << 16;
    float *xm = reinterpret_cast<float *>(smem + C::kXOff);  // [k][h][128]
    // c = scale * log2(e), times the descale factors of Q and K for e4m3 inputs.
    const float c = FP8 ? p.scale_log2 * p.descale_q[bh] * p.descale_k[bh] : p.scale_log2;
    const uint64_t c2 = f2pack(c, c);
    float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f}, lr[2] = {0.f, 0.f};
    const int n_k[2] = {n_kv0, n_kv1};
    bool ok = !*abort_flag;
    for (int j = 0; j < n_kv && ok; ++j) {
      for (int k = 0; k < 2 && ok; ++k) {
        if (j >= n_k[k]) continue;
        const int qt = 2 * u + k;
        const uint32_t tS = tmem + lane_off + 128 * k + 64 * h;
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_s_full[k], j & 1, kTagSFull));
        if (!ok) break;
        tc_fence_after();
        if (r == 0 && h == 0) FA_TRACE(528 + k * 256 + 4 * j + 0);
        uint32_t s[64];
        tmem_ld32(tS, s);
        tmem_ld32(tS + 32, s + 32);
        tmem_wait_ld();
        // Keys j*128 + 64h + col are valid when col < nv (tail of N, causal diagonal).
        int nvalid = min(128, p.N - j * 128);
        if (CAUSAL && j == qt) nvalid = min(nvalid, r + 1);
        const int nv = nvalid - 64 * h;
        if (nv < 64) {
#pragma unroll
          for (int cc = 0; cc < 64; ++cc)
            if (cc >= nv) s[cc] = __float_as_uint(-INFINITY);
        }
        // Dropout: keep bit cc for key j*128 + 64h + cc of query row qt*128 + r,
        // eight keys per generator call (the counter's key block).
        uint64_t keep = ~0ull;
        if constexpr (DROPOUT) {
          keep = 0;
          const uint32_t jb0 = static_cast<uint32_t>(j * 128 + 64 * h) >> 3;
#pragma unroll
          for (int t = 0; t < 8; ++t)
            keep |= static_cast<uint64_t>(dropout_keep8(p.drop, qt * 128 + r, jb0 + t, bh)) << (8 * t);
        }
        // Half-row max as a shallow tree (eight independent chains of four).
        float mq[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          const float *v = reinterpret_cast<const float *>(s + 8 * q);
          mq[q] = fmaxf(fmax3(fmax3(fmax3(v[0], v[1], v[2]), v[3], v[4]), v[5], v[6]), v[7]);
        }
        const float mh = fmax3(fmax3(mq[0], mq[1], mq[2]), fmax3(mq[3], mq[4], mq[5]), fmaxf(mq[6], mq[7]));
        xm[(k * 2 + h) * 128 + r] = mh;
        mbar_arrive(&bar_x[k * 4 + rq]);
        // P = 2^(c*S - m) for this half row, with the row sums of P in fp32
        // (for the LSE) and of P rounded to bf16 (the PV weights; O's normaliser).
        uint32_t pk[32];
        float psum = 0.f, prsum = 0.f;
        auto exps = [&](float mref) {
          const float neg = (mref == -INFINITY) ? 0.f : -mref;
          const uint64_t n2 = f2pack(neg, neg);
          if constexpr (FP8) {
            // P rounded to e4m3, four keys per word; O's normaliser is the fp32
            // sum of the unrounded P (the same sum as the LSE's).
            uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int cq = 0; cq < 16; ++cq) {
              const uint64_t xa = ffma2(f2pack(__uint_as_float(s[4 * cq]), __uint_as_float(s[4 * cq + 1])), c2, n2);
              const uint64_t xb =
                  ffma2(f2pack(__uint_as_float(s[4 * cq + 2]), __uint_as_float(s[4 * cq + 3])), c2, n2);
              float x0, x1, x2, x3;
              f2unpack(xa, x0, x1);
              f2unpack(xb, x2, x3);
              const float a0 = ex2(x0), a1 = ex2(x1), a2 = ex2(x2), a3 = ex2(x3);
              acc[cq & 3] = fadd2(acc[cq & 3], fadd2(f2pack(a0, a1), f2pack(a2, a3)));
              pk[cq] = pack_e4m3x4(a0, a1, a2, a3);
            }
            float u0, u1, u2, u3, u4, u5, u6, u7;
            f2unpack(acc[0], u0, u1);
            f2unpack(acc[1], u2, u3);
            f2unpack(acc[2], u4, u5);
            f2unpack(acc[3], u6, u7);
            psum = ((u0 + u1) + (u2 + u3)) + ((u4 + u5) + (u6 + u7));
            prsum = psum;
            return;
          }
          uint64_t acc[2] = {0ull, 0ull}, racc[2] = {0ull, 0ull};
#pragma unroll
          for (int cc = 0; cc < 32; ++cc) {
            const uint64_t x2 = ffma2(f2pack(__uint_as_float(s[2 * cc]), __uint_as_float(s[2 * cc + 1])), c2, n2);
            float x0, x1;
            f2unpack(x2, x0, x1);
            const float a = ex2(x0), b = ex2(x1);
            acc[cc & 1] = fadd2(acc[cc & 1], f2pack(a, b));
            const uint32_t w = pack_bf16(a, b);
            // The sums are of P before dropout; the PV product takes the kept entries
            // (the 1/keep-probability scale is applied to O in the epilogue).
            pk[cc] = DROPOUT ? (w & keep_pair_mask(keep, cc)) : w;
            racc[cc & 1] = fadd2(racc[cc & 1], f2pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
          }
          float u0, u1, u2, u3, v0, v1, v2, v3;
          f2unpack(acc[0], u0, u1);
          f2unpack(acc[1], u2, u3);
          f2unpack(racc[0], v0, v1);
          f2unpack(racc[1], v2, v3);
          psum = (u0 + u1) + (u2 + u3);
          prsum = (v0 + v1) + (v2 + v3);
        };
        const float m_old = m[k];
        if (m_old != -INFINITY) exps(m_old);  // optimistic: the running max usually holds
        ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_x[k * 4 + rq], j & 1, kTagXmax));
        if (!ok) break;
        const float m_cand = fmaxf(mh, xm[(k * 2 + (h ^ 1)) * 128 + r]) * c;
        float alpha = 1.f;
        bool rescale = false;
        if (m_cand > m_old + 8.f) {  // also taken on the first tile (m = -inf)
          alpha = ex2(m_old - m_cand);
          rescale = (m_old != -INFINITY);
          m[k] = m_cand;
          exps(m_cand);
        }
        l[k] = l[k] * alpha + psum;
        lr[k] = lr[k] * alpha + prsum;
        if (__any_sync(0xffffffffu, rescale)) {
          // O_k still holds the previous step's PV: wait for it, then rescale
          // this warp's column half of O.
          ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_pv_done[k], (j - 1) & 1, kTagPvDone));
          if (!ok) break;
          tc_fence_after();
          const uint32_t tO = tmem + lane_off + 256 + k * D + h * (D / 2);
#pragma unroll
          for (int ch = 0; ch < D / 64; ++ch) {
            uint32_t o[32];
            tmem_ld32(tO + ch * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * alpha);
            tmem_st32(tO + ch * 32, o);
          }
        }
        if constexpr (FP8)
          tmem_st16(tS, pk);  // 64 keys of e4m3 P in 16 columns
        else
          tmem_st32(tS, pk);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&bar_p_full[k]);
        if (r == 0 && h == 0) FA_TRACE(528 + k * 256 + 4 * j + 1);
        if (lane == 0 && j < 16) FA_TRACE(1024 + (k * 8 + warp) * 16 + j);
      }
    }
    // ---------------------------------------------------------- epilogue
    // Once both tiles' last PV has completed no MMA or load is in flight, so the
    // K/V ring is free.  Each warp converts its 32 rows x D/2 columns of O_k (and
    // their rounding residual) to bf16, stages them in its own 2 x 32 x D bytes
    // of the ring and writes them out with plain coalesced stores: a warp-wide
    // 16-byte access covers whole D-byte row segments.  Nothing waits for the
    // stores, so the CTA can exit (and the next CTA start) as soon as they issue.
    ok = ok && __all_sync(0xffffffffu, mbar_wait(ctx, &bar_pv_done[0], (n_k[0] - 1) & 1, kTagPvDone) &&
                                           mbar_wait(ctx, &bar_pv_done[1], (n_k[1] - 1) & 1, kTagPvDone));
    if (ok) tc_fence_after();
    constexpr int kChunks = D / 16;         // 16-byte chunks in a row's D/2 bf16 columns
    constexpr int kRowsPerPass = 512 / D;   // rows covered by one warp-wide 16-byte access
    const uint32_t scr_o = smem_u32(sKV) + warp * (2 * 32 * D);
    const uint32_t scr_lo = scr_o + 32 * D;
    for (int k = 0; k < 2 && ok; ++k) {
      const int qt = 2 * u + k;
      // Whole-row sums from the two column halves.
      float *ls = reinterpret_cast<float *>(smem + C::kLOff) + k * 512;  // [h][2][128]
      ls[(h * 2 + 0) * 128 + r] = l[k];
      ls[(h * 2 + 1) * 128 + r] = lr[k];
      mbar_arrive(&bar_l[k * 4 + rq]);
      ok = __all_sync(0xffffffffu, mbar_wait(ctx, &bar_l[k * 4 + rq], 0, kTagLsum));
      if (!ok) break;
      if (r == 0 && h == 0) FA_TRACE(4 + k);
      const float lt = l[k] + ls[((h ^ 1) * 2 + 0) * 128 + r];
      const float lrt = lr[k] + ls[((h ^ 1) * 2 + 1) * 128 + r];
      const float inv_l = (FP8 ? p.descale_v[bh] : (DROPOUT ? p.drop.inv_keep : 1.f)) / lrt;
      const uint32_t tO = tmem + lane_off + 256 + k * D + h * (D / 2);
      uint32_t o[D / 2];
#pragma unroll
      for (int ch = 0; ch < D / 64; ++ch) tmem_ld32(tO + 32 * ch, o + 32 * ch);
      tmem_wait_ld();
      uint32_t w[D / 4];
#pragma unroll
      for (int t = 0; t < D / 4; ++t)
        w[t] = pack_bf16(__uint_as_float(o[2 * t]) * inv_l, __uint_as_float(o[2 * t + 1]) * inv_l);
#pragma unroll
      for (int c = 0; c < kChunks; ++c)
        st_shared_v4(scr_o + epi_offset<D>(lane, c), w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      if (p.o_lo != nullptr) {
        // What rounding O to bf16 dropped, itself rounded to bf16: O ~ o + o_lo
        // to about 16 significant bits (used by the backward's D = rowsum(dO o O)).
#pragma unroll
        for (int t = 0; t < D / 4; ++t) {
          const float a = __uint_as_float(o[2 * t]) * inv_l, b = __uint_as_float(o[2 * t + 1]) * inv_l;
          w[t] = pack_bf16(a - __uint_as_float(w[t] << 16), b - __uint_as_float(w[t] & 0xFFFF0000u));
        }
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
          st_shared_v4(scr_lo + epi_offset<D>(lane, c), w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
      }
      __syncwarp();
      // Row rq*32 + row of query tile qt; lane reads chunk c of its row.
      const int c = lane % kChunks;
      const int row0 = qt * 128 + rq * 32;
#pragma unroll
      for (int pass = 0; pass < 32 / kRowsPerPass; ++pass) {
        const int row = pass * kRowsPerPass + lane / kChunks;
        if (row0 + row < p.N) {
          const size_t e = (static_cast<size_t>(bh) * p.N + row0 + row) * D + h * (D / 2) + c * 8;
          *reinterpret_cast<uint4 *>(p.o + e) = ld_shared_u4(scr_o + epi_offset<D>(row, c));
          if (p.o_lo != nullptr) *reinterpret_cast<uint4 *>(p.o_lo + e) = ld_shared_u4(scr_lo + epi_offset<D>(row, c));
        }
      }
      __syncwarp();  // the next tile rewrites this warp's staging
      const int grow = qt * 128 + r;
      if (h == 0 && grow < p.N) p.lse[static_cast<size_t>(bh) * p.N + grow] = (m[k] + log2f(lt)) * 0.69314718055994531f;
    }
    if (ok && threadIdx.x == 0) FA_TRACE(6);
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (threadIdx.x == 0) FA_TRACE(7);
  if (warp == C::kIssuerWarp) tmem_dealloc(tmem, 512);
}

}  // namespace fa
