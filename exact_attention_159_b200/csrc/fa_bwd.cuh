// fa_bwd.cuh -- backward exact attention on sm_100a.
//
// P is recomputed from the saved log-sum-exp instead of being stored
// ("NVIDIA Blackwell: FlashAttention-4 Overcomes Memory Bottlenecks": the
// backward keeps its intermediates in tensor memory rather than shared
// memory, which cuts shared-memory traffic).  Three
// kernels run on the caller's stream:
//   bwd_prep_kernel    D_i = dO_i . O_i, LSE2_i = LSE_i * log2(e) (+inf on the
//                      padding rows of the last tile), dQ_acc = 0
//   bwd_kernel         one CTA per (batch * key/value head, 128-row key tile n),
//                      key tile stationary, loop over the query tiles m that see
//                      it, of every query head that reads this key/value head
//                      (grouped-query attention sums their dK, dV in TMEM):
//                        S^T  = K_n Q_m^T                 (tcgen05 -> TMEM)
//                        P^T  = 2^(S^T scale log2e - LSE2) (CUDA cores -> TMEM, bf16)
//                        dP^T = V_n dO_m^T                (tcgen05 -> TMEM)
//                        dS^T = P^T (dP^T - D)            (CUDA cores -> smem and TMEM, bf16)
//                        dV  += P^T dO_m                  (A from TMEM)
//                        dK  += dS^T Q_m                  (A from TMEM)
//                        dQ_m = dS K_n                    (A from smem; TMEM) -> fp32 TMA reduce-add
//                                                          into dQ_acc
//                      dK (x scale) and dV leave TMEM once, at the end.
//   bwd_dq_kernel      dQ = bf16(scale * dQ_acc)
// Warps: 0 TMA producer, 1 MMA issuer + TMEM owner, 2..5 P/dS for the 128 key
// rows (thread = key row), 6..9 dQ drain (thread = query row).
// Tensor memory columns: dK [0,D), dV [D,2D), S^T [2D,2D+128),
// dP^T [2D+128,2D+256) with dS^T (bf16, packed two per column) written over
// its first 64 columns once they have been read; dQ reuses the dP^T columns
// when D = 128 (the 512 columns are otherwise full; dK, issued first, has read
// dS^T by then) and has its own 64 columns when D = 64.
#pragma once

#include "fa_fwd.cuh"

namespace fa {

struct BwdParams {
  const float* nlse2;  // [B * Hq, Npad]  -LSE * log2(e); -inf on padding rows and rows that see no key
  const float* ndsum;  // [B * Hq, Npad]  -D_i, 0 on padding rows
  __nv_bfloat16* dK;   // [B * Hkv, Nk, D]  (bf16 outputs, when dK_acc is null)
  __nv_bfloat16* dV;   // [B * Hkv, Nk, D]
  float* dK_acc;       // [B * Hkv, Nk, D] fp32 accumulators: when set, dK (x scale) and dV are added
  float* dV_acc;       // to them (or stored, when acc_first) instead of written as bf16
  int acc_first;
  int N, Npad;         // query rows per head, padded to whole tiles
  int Nk;              // key rows per head
  int BHkv, Hq, Hkv, G;  // batch * key/value heads; heads per batch entry; query heads per key/value head
  int off;             // Nk - N: query row i sees keys j <= i + off when causal
  int n_q_tiles, n_kv_tiles;
  float scale_log2;    // scale * log2(e)
  float scale;
  int* status;
};

template <int D>
struct BwdLayout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kK = 0;
  static constexpr int kV = kK + kTileBytes;
  static constexpr int kQ = kV + kTileBytes;        // two stages
  static constexpr int kdO = kQ + 2 * kTileBytes;   // one stage
  static constexpr int kdS = kdO + kTileBytes;      // dS^T, 128 x 128 bf16, two 64-column chunks
  static constexpr int kDQ = kdS + 32768;           // two 16 KB staging buffers: 128 rows x 32 fp32 of dQ
  static constexpr int kLse = kDQ + 32768;          // two stages of 128 fp32 (-LSE2)
  static constexpr int kDsum = kLse + 1024;         // two stages of 128 fp32 (-D)
  static constexpr int kBar = kDsum + 1024;
  // kv_full, q_full[2], q_empty[2], do_full, do_empty, s_full, dp_full, p_full, ds_full, ds_empty,
  // dq_full, dq_free, acc_full, drain
  static constexpr int kNumBars = 16;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kNeed = kMisc + 16;           // the dynamic shared memory base is 1024-byte aligned
  // Keep one CTA per SM (each CTA allocates all 512 TMEM columns).
  static constexpr int kBytes = kNeed > 120 * 1024 ? kNeed : 120 * 1024;
  static constexpr bool kAliasDQ = (D == 128);
  static constexpr uint32_t kColDK = 0, kColDV = D, kColS = 2 * D, kColDP = 2 * D + 128;
  static constexpr uint32_t kColDQ = kAliasDQ ? kColDP : 2 * D + 256;
  static constexpr int kThreads = 384;  // 12 warps: control, P/dS, dQ drain
};

// Register split (setmaxnreg): 128 * (80 + 240 + 184) = 384 * 168, the launch's total.  Each
// setmaxnreg heads its role's branch so the register budget of that code is unambiguous.
constexpr int kBwdRegsCtl = 80, kBwdRegsP = 240, kBwdRegsDQ = 184;
constexpr int kBwdLaunchRegs = (65536 / 384) / 8 * 8;  // per-thread registers at launch (384 threads)
static_assert(128 * (kBwdRegsCtl + kBwdRegsP + kBwdRegsDQ) <= 384 * kBwdLaunchRegs,
              "backward register split exceeds the launch's registers");

// GEN: grouped-query heads and / or Nq != Nk; without it (one query head per key/value head,
// Nq == Nk) the group and offset terms are compile-time constants.
template <int D, bool CAUSAL, int POLY16, bool GEN>
__global__ void __launch_bounds__(384, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmdO,
               const __grid_constant__ CUtensorMap tmdQacc, const BwdParams prm) {
  using L = BwdLayout<D>;
  constexpr int T = L::kTileBytes;
  constexpr int kChunks = D / 64;

  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicCAS(prm.status, 0, kSiteBwd | 0x7F);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t *kv_full = bars + 0, *q_full = bars + 1, *q_empty = bars + 3, *do_full = bars + 5;
  uint64_t *do_empty = bars + 6, *s_full = bars + 7, *dp_full = bars + 8, *p_full = bars + 9;
  uint64_t *ds_full = bars + 10, *ds_empty = bars + 11, *dq_full = bars + 12, *dq_free = bars + 13;
  uint64_t *acc_full = bars + 14, *drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int off = GEN ? prm.off : 0;
  const int Nk = GEN ? prm.Nk : prm.N;
  int bkv, n;  // key tile n = 0 (the most causal work) first, a few heads at a time
  cta_order(blockIdx.x, prm.BHkv, prm.n_kv_tiles, cta_head_group(prm.BHkv, prm.n_kv_tiles, CAUSAL), bkv, n);
  // first query tile that sees key tile n: its last row + off reaches the tile's first key
  int m_begin = 0;
  if (CAUSAL) {
    const int r0 = n * kTile - off;  // first query row that sees key n * kTile
    m_begin = !GEN ? n : r0 <= 0 ? 0 : r0 / kTile;
  }
  const int n_m = prm.n_q_tiles - m_begin;      // >= 1: every real key is seen by the last query row
  const int n_it = GEN ? prm.G * n_m : n_m;     // (query head of the group, query tile) pairs
  const int bq0 = GEN ? (bkv / prm.Hkv) * prm.Hq + (bkv % prm.Hkv) * prm.G : bkv;  // first query head of the group

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(&q_full[st], 1);
      mbar_init(&q_empty[st], 1);
    }
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 128);
    mbar_init(ds_full, 128);
    mbar_init(ds_empty, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 128);
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Guard g{abort_flag, prm.status};

  if (warp < 4) {
    regs_to<kBwdRegsCtl, kBwdLaunchRegs>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmdO);
        mbar_expect_tx(kv_full, 2 * T);
        for (int c = 0; c < kChunks; ++c) {
          tma_load_3d(smem + L::kK + c * 16384, &tmK, 64 * c, n * kTile, bkv, kv_full);
          tma_load_3d(smem + L::kV + c * 16384, &tmV, 64 * c, n * kTile, bkv, kv_full);
        }
        bool ok = true;
        int q_issued = 0, do_issued = 0;
        for (int it = 0; it < n_it; ++it) {
          const int bq = GEN ? bq0 + it / n_m : bq0, m = GEN ? m_begin + it % n_m : m_begin + it, st = it & 1;
          // Q_m, -LSE2_m, -D_m into stage st (two stages)
          if (!(ok = wait(&q_empty[st], ((it >> 1) & 1) ^ 1, g, kSiteBwd | 1))) break;
          mbar_expect_tx(&q_full[st], T + 1024);
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(smem + L::kQ + st * T + c * 16384, &tmQ, 64 * c, m * kTile, bq, &q_full[st]);
          const size_t off = static_cast<size_t>(bq) * prm.Npad + static_cast<size_t>(m) * kTile;
          bulk_load(smem + L::kLse + 512 * st, prm.nlse2 + off, 512, &q_full[st]);
          bulk_load(smem + L::kDsum + 512 * st, prm.ndsum + off, 512, &q_full[st]);
          ++q_issued;
          // dO_m (one stage: free once dV_{m-1} has read it)
          if (!(ok = wait(do_empty, (it & 1) ^ 1, g, kSiteBwd | 14))) break;
          mbar_expect_tx(do_full, T);
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(smem + L::kdO + c * 16384, &tmdO, 64 * c, m * kTile, bq, do_full);
          ++do_issued;
        }
        if (!ok) {
          drain_wait(kv_full, 0);
          for (int i = q_issued - 2 > 0 ? q_issued - 2 : 0; i < q_issued; ++i)
            drain_wait(&q_full[i & 1], (i >> 1) & 1);
          if (do_issued > 0) drain_wait(do_full, (do_issued - 1) & 1);
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------------- MMA
      // Issue order per query tile m: dP_m, dV_m, S_{m+1}, dK_m, dQ_m -- S of the next tile is
      // computed while the softmax warps turn dP_m into dS_m.
      if (lane == 0) {
        constexpr uint32_t idKK = idesc_bf16_f32(128, 128, false, false);  // S^T, dP^T: both K-major
        constexpr uint32_t idKM = idesc_bf16_f32(128, D, false, true);     // dV (A in TMEM), dK: B MN-major
        constexpr uint32_t idMM = idesc_bf16_f32(128, D, true, true);      // dQ: A and B MN-major
        const uint32_t sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
        const uint32_t sQ0 = smem_u32(smem + L::kQ), sdO = smem_u32(smem + L::kdO);
        const uint32_t sdS = smem_u32(smem + L::kdS);
        auto issue_s = [&](int st) {  // S^T = K Q^T
          const uint32_t sQ = sQ0 + st * T;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss(tmem + L::kColS, sdesc_sw128(sK + off, 16, 1024), sdesc_sw128(sQ + off, 16, 1024), idKK,
                   kk > 0);
          }
          tc_commit(s_full);
        };
        bool ok = wait(kv_full, 0, g, kSiteBwd | 2) && wait(&q_full[0], 0, g, kSiteBwd | 3);
        if (ok) {
          tc_fence_after();
          issue_s(0);
        }
        for (int it = 0; ok && it < n_it; ++it) {
          const int st = it & 1;
          const uint32_t ph = it & 1;
          const uint32_t sQ = sQ0 + st * T;
          // dP^T = V dO^T (its columns hold dQ of the previous tile when aliased)
          if (!(ok = wait(do_full, ph, g, kSiteBwd | 15))) break;
          if (L::kAliasDQ && it > 0) {
            if (!(ok = wait(dq_free, ph ^ 1, g, kSiteBwd | 4))) break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            mma_ss(tmem + L::kColDP, sdesc_sw128(sV + off, 16, 1024), sdesc_sw128(sdO + off, 16, 1024), idKK,
                   kk > 0);
          }
          tc_commit(dp_full);
          // dV += P^T dO
          if (!(ok = wait(p_full, ph, g, kSiteBwd | 5))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(tmem + L::kColDV, tmem + L::kColS + 8 * kk, sdesc_sw128(sdO + kk * 2048, 16384, 1024), idKM,
                   (it > 0 || kk > 0) ? 1u : 0u);
          tc_commit(do_empty);
          // S^T of the next query tile (P_m in the S columns has been read by the dV MMA above)
          if (it + 1 < n_it) {
            if (!(ok = wait(&q_full[st ^ 1], ((it + 1) >> 1) & 1, g, kSiteBwd | 16))) break;
            tc_fence_after();
            issue_s(st ^ 1);
          }
          // dK += dS^T Q (dS^T from TMEM, over the dP^T columns)
          if (!(ok = wait(ds_full, ph, g, kSiteBwd | 6))) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(tmem + L::kColDK, tmem + L::kColDP + 8 * kk, sdesc_sw128(sQ + kk * 2048, 16384, 1024), idKM,
                   (it > 0 || kk > 0) ? 1u : 0u);
          tc_commit(&q_empty[st]);  // Q_m, -LSE2_m, -D_m no longer needed once these land
          // dQ_m = dS K
          if (!L::kAliasDQ && it > 0) {
            if (!(ok = wait(dq_free, ph ^ 1, g, kSiteBwd | 7))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ss(tmem + L::kColDQ, sdesc_sw128(sdS + kk * 2048, 16384, 1024),
                   sdesc_sw128(sK + kk * 2048, 16384, 1024), idMM, kk > 0);
          tc_commit(dq_full);
          tc_commit(ds_empty);
        }
        if (ok) tc_commit(acc_full);
        tc_commit(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (warp < 8) {
    regs_to<kBwdRegsP, kBwdLaunchRegs>();
    // --------------------------------------------------- P^T and dS^T rows
    const int quarter = warp & 3;
    const int j = quarter * 32 + lane;  // key row within the tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + L::kColS + lane_off, tdP = tmem + L::kColDP + lane_off;
    uint8_t* sdS = smem + L::kdS;
    const float2 c2 = make_float2(prm.scale_log2, prm.scale_log2);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int m = GEN ? m_begin + it % n_m : m_begin + it, st = it & 1;
      const uint32_t ph = it & 1;
      const float4* nl4 = reinterpret_cast<const float4*>(smem + L::kLse + 512 * st);
      const float4* nd4 = reinterpret_cast<const float4*>(smem + L::kDsum + 512 * st);
      // -LSE2_m / -D_m arrive with Q_m (TMA); S^T_m is ready once s_full completes
      if (!(ok = wait_warp(&q_full[st], (it >> 1) & 1, g, kSiteBwd | 13))) break;
      if (!(ok = wait_warp(s_full, ph, g, kSiteBwd | 8))) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sr[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(sr[c]);
      float p[kTile];
      // causal masking in this pair of tiles: query i (of tile m) does not see key j (of tile n)
      // when n*128 + j > m*128 + i + off, i.e. i < thr
      const int thr = GEN ? (n - m) * kTile + j - off : j;
      const bool diag = CAUSAL && (GEN ? n * kTile + kTile - 1 > m * kTile + off : m == n);
      const bool edge = diag || (m + 1) * kTile > prm.N;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const int i = 32 * cc + 4 * e4;
          const float4 nl = nl4[i >> 2];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int ii = i + 2 * h;
            const float2 x =
                __ffma2_rn(make_float2(__uint_as_float(sr[cc][ii & 31]), __uint_as_float(sr[cc][(ii + 1) & 31])), c2,
                           h == 0 ? make_float2(nl.x, nl.y) : make_float2(nl.z, nl.w));
            float2 pv;
            if (!edge && ((ii >> 1) & 7) < POLY16 / 2) {
              pv = exp2_poly2(x);
            } else {
              pv.x = exp2_sfu(x.x);
              pv.y = exp2_sfu(x.y);
              if (diag) {
                if (ii < thr) pv.x = 0.0f;
                if (ii + 1 < thr) pv.y = 0.0f;
              }
            }
            p[ii] = pv.x;
            p[ii + 1] = pv.y;
            pk[(ii & 31) >> 1] = pack_bf16x2(pv.x, pv.y);
          }
        }
        tmem_st16(tS + 16 * cc, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(p_full);

      if (!(ok = wait_warp(dp_full, ph, g, kSiteBwd | 9))) break;
      tc_fence_after();
      if (it > 0) {
        if (!(ok = wait_warp(ds_empty, ph ^ 1, g, kSiteBwd | 10))) break;
      }
      uint32_t dp_[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if ((c & 1) == 0) {  // dP^T columns 64 at a time
          tmem_ld32(tdP + 32 * c, dp_[0]);
          tmem_ld32(tdP + 32 * c + 32, dp_[1]);
          tmem_wait_ld();
          reg_fence(dp_[0]);
          reg_fence(dp_[1]);
        }
        uint32_t(&dpc)[32] = dp_[c & 1];
        uint32_t w[16];
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const int i = 32 * c + 4 * e4;
          const float4 nd = nd4[i >> 2];
          const float2 t0 = __fadd2_rn(
              make_float2(__uint_as_float(dpc[4 * e4]), __uint_as_float(dpc[4 * e4 + 1])), make_float2(nd.x, nd.y));
          const float2 t1 =
              __fadd2_rn(make_float2(__uint_as_float(dpc[4 * e4 + 2]), __uint_as_float(dpc[4 * e4 + 3])),
                         make_float2(nd.z, nd.w));
          const float2 d0 = __fmul2_rn(make_float2(p[i], p[i + 1]), t0);
          const float2 d1 = __fmul2_rn(make_float2(p[i + 2], p[i + 3]), t1);
          w[2 * e4] = pack_bf16x2(d0.x, d0.y);
          w[2 * e4 + 1] = pack_bf16x2(d1.x, d1.y);
        }
        // columns 32c .. 32c+31 live in chunk (32c / 64), 16-byte groups 4*(c&1) .. +3
        // dS^T to TMEM for dK, over dP^T columns already read (block c lands in columns 16c..16c+15)
        tmem_st16(tdP + 16 * c, w);
        uint8_t* base = sdS + (c >> 1) * 16384;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t col = (c & 1) * 32 + q4 * 8;
          *reinterpret_cast<uint4*>(base + sw128_offset(j, col)) =
              make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
        }
      }
      fence_proxy_async();
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(ds_full);
    }
    if (ok) ok = wait_warp(acc_full, 0, g, kSiteBwd | 11);
    if (ok) {
      tc_fence_after();
      const int key = n * kTile + j;
      const bool store = key < Nk;
      const size_t rowoff = (static_cast<size_t>(bkv) * Nk + (store ? key : 0)) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tcol = tmem + (which == 0 ? L::kColDK : L::kColDV) + lane_off;
        const float mul = which == 0 ? prm.scale : 1.0f;
        if (prm.dK_acc != nullptr) {
          // fp32 accumulators (gradients of one query block summed over several calls); each key
          // row belongs to exactly one CTA, so the read-modify-write needs no atomics
          float* acc_row = (which == 0 ? prm.dK_acc : prm.dV_acc) + rowoff;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t a[32];
            tmem_ld32(tcol + 32 * c, a);
            tmem_wait_ld();
            reg_fence(a);
            if (store) {
              float4* dst = reinterpret_cast<float4*>(acc_row + 32 * c);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                float4 v = make_float4(__uint_as_float(a[4 * i]) * mul, __uint_as_float(a[4 * i + 1]) * mul,
                                       __uint_as_float(a[4 * i + 2]) * mul, __uint_as_float(a[4 * i + 3]) * mul);
                if (!prm.acc_first) {
                  const float4 o = dst[i];
                  v.x += o.x;
                  v.y += o.y;
                  v.z += o.z;
                  v.w += o.w;
                }
                dst[i] = v;
              }
            }
          }
          continue;
        }
        __nv_bfloat16* dst_row = (which == 0 ? prm.dK : prm.dV) + rowoff;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t a[32];
          tmem_ld32(tcol + 32 * c, a);
          tmem_wait_ld();
          reg_fence(a);
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            w[i] = pack_bf16x2(__uint_as_float(a[2 * i]) * mul, __uint_as_float(a[2 * i + 1]) * mul);
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(dst_row + 32 * c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
          }
        }
      }
    }
  } else {
    regs_to<kBwdRegsDQ, kBwdLaunchRegs>();
    // ---------------------------------------------------------- dQ drain
    // dQ_m (fp32, in TMEM) leaves 32 columns at a time through a swizzled shared-memory staging
    // buffer and a TMA reduce-add into the fp32 accumulator (two buffers, ping-pong).
    const int quarter = warp & 3;
    const int i = quarter * 32 + lane;  // query row within the tile
    const bool leader = (warp == 8 && lane == 0);
    const uint32_t tdQ = tmem + L::kColDQ + (static_cast<uint32_t>(quarter * 32) << 16);
    uint8_t* stage0 = smem + L::kDQ;
    if (leader) prefetch_tmap(&tmdQacc);
    // The four drain warps pass the same hardware barriers (id 1) in the same order; the only
    // wait that can fail (dq_full) is followed by a joint decision, so they leave together.
    int flushed = 0;  // quarter tiles handed to TMA so far
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int bq = GEN ? bq0 + it / n_m : bq0, m = GEN ? m_begin + it % n_m : m_begin + it;
      const bool okl = ok && wait_warp(dq_full, it & 1, g, kSiteBwd | 12);
      if (!(ok = group_and(1, 128, okl))) break;
      tc_fence_after();
      uint32_t a[D / 32][32];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) tmem_ld32(tdQ + 32 * c, a[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) reg_fence(a[c]);
      tc_fence_before();
      mbar_arrive(dq_free);  // the dQ columns may be overwritten now
#pragma unroll
      for (int c = 0; c < D / 32; ++c, ++flushed) {
        uint8_t* buf = stage0 + (flushed & 1) * 16384;
        if (leader) bulk_wait_read<1>();  // the reduce that last used this buffer has read it
        named_barrier(1, 128);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          *reinterpret_cast<uint4*>(buf + i * 128 + (((v ^ i) & 7) << 4)) =
              make_uint4(a[c][4 * v], a[c][4 * v + 1], a[c][4 * v + 2], a[c][4 * v + 3]);
        fence_proxy_async();
        named_barrier(1, 128);
        if (leader) {
          tma_reduce_add_3d(&tmdQacc, 32 * c, m * kTile, bq, buf);
          bulk_commit();
        }
      }
    }
    if (leader) bulk_wait<0>();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// -D_i = -sum_c dO_ic O_ic (fp32 from bf16), -LSE2_i = -LSE_i log2(e), dQ_acc = 0.
// Rows i >= N of the padded last tile get D = 0 and LSE2 = +inf (so P = 0 there).
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const __nv_bfloat16* __restrict__ O,
                                                       const __nv_bfloat16* __restrict__ dO,
                                                       const float* __restrict__ LSE, float* __restrict__ nlse2,
                                                       float* __restrict__ ndsum, float* __restrict__ dq_acc, int N,
                                                       int Npad, long long rows_total) {
  constexpr int G = D / 8;  // threads per row, 8 elements (16 bytes) each
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long r = t / G;
  const int seg = static_cast<int>(t % G);
  const bool live = r < rows_total;
  const long long bh = live ? r / Npad : 0;
  const int i = live ? static_cast<int>(r % Npad) : 0;
  const bool valid = live && i < N;
  float acc = 0.0f;
  if (valid) {
    const size_t e = (static_cast<size_t>(bh) * N + i) * D + seg * 8;
    const uint4 a = *reinterpret_cast<const uint4*>(O + e);
    const uint4 b = *reinterpret_cast<const uint4*>(dO + e);
    const __nv_bfloat162* pa = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&b);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 fa = __bfloat1622float2(pa[k]), fb = __bfloat1622float2(pb[k]);
      acc = fmaf(fa.x, fb.x, acc);
      acc = fmaf(fa.y, fb.y, acc);
    }
  }
#pragma unroll
  for (int off = G / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (live) {
    if (seg == 0) {
      ndsum[r] = valid ? -acc : 0.0f;
      const float lse = valid ? LSE[static_cast<size_t>(bh) * N + i] : -INFINITY;
      nlse2[r] = lse == -INFINITY ? -INFINITY : -lse * 1.4426950408889634f;  // -inf: no key seen, P = 0
    }
    float4* z = reinterpret_cast<float4*>(dq_acc + r * D + seg * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

// dQ = bf16(scale * dQ_acc) for the N real rows of every head.
template <int D>
__global__ void __launch_bounds__(256) bwd_dq_kernel(const float* __restrict__ dq_acc,
                                                     __nv_bfloat16* __restrict__ dQ, float scale, int N, int Npad,
                                                     long long rows_total) {
  constexpr int G = D / 8;
  const long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long r = t / G;  // over BH * N real rows
  const int seg = static_cast<int>(t % G);
  if (r >= rows_total) return;
  const long long bh = r / N;
  const int i = static_cast<int>(r % N);
  const float4* src = reinterpret_cast<const float4*>(dq_acc + (bh * Npad + i) * D + seg * 8);
  const float4 a = src[0], b = src[1];
  uint4 o;
  o.x = pack_bf16x2(a.x * scale, a.y * scale);
  o.y = pack_bf16x2(a.z * scale, a.w * scale);
  o.z = pack_bf16x2(b.x * scale, b.y * scale);
  o.w = pack_bf16x2(b.z * scale, b.w * scale);
  *reinterpret_cast<uint4*>(dQ + r * D + seg * 8) = o;
}

}  // namespace fa
