// fa_bwd2.cuh -- backward exact attention on a cluster pair of SMs (2-CTA UMMA), d = 128.
//
// The FlashAttention-4 pages describe the backward pass on CTA pairs that share one large tile,
// each carrying half of the operands and passing intermediate results to the other without a
// trip to HBM ("C. Le Duo de Cuisiniers (2-CTA)").  Here a cluster of two CTAs owns the two
// adjacent key tiles n0 = 2u (rank 0) and n1 = 2u + 1 (rank 1) of one head and loops over the
// query tiles m that see them.  Per query tile, with every MMA a tcgen05.mma.cta_group::2 issued
// by rank 0 for both SMs:
//   S^T  = K Q_m^T        M = 256 (each CTA its own 128 keys), B = Q_m split by query rows
//   dP^T = V dO_m^T       the same shape
//   dV  += P^T dO_m       A (P^T, bf16) from tensor memory, B = dO_m split by columns of d
//   dK  += dS^T Q_m       A (dS^T, bf16) from tensor memory, B = Q_m split by columns of d
//   dQ_m = dS [K_n0; K_n1]  M = 128 (each CTA 64 query rows) over the pair's 256 keys: each CTA
//                        hands the other the half of its dS^T that the other's query rows need
//                        (shared memory of the peer, written directly), so dQ of a query tile
//                        is summed over two key tiles before it leaves the chip
// Against the single-CTA kernel every B operand is read half by each SM, and the dQ drain
// (TMEM -> shared memory -> TMA reduce-add) moves half as much per SM: about 350 KB of
// shared-memory traffic per SM and query tile instead of about 500 KB.  Measured on B200 it is
// nevertheless slower than the single-CTA kernel: at N = 128 the 16 M = 128 dQ instructions cost
// more than the single-CTA kernel's 8, and the remote dS stores with their release cost the dS
// warps 2,000-3,000 clocks per tile, on which the MMA issuer then waits.  It is selected only on
// request.
//
// Operand placement.  In a pair MMA the rows of A come half from each CTA while B is one matrix
// split by columns between the two, so every slice of the contraction must hold the same
// indices in both CTAs, at the same shared-memory (or tensor-memory) offset.  Each CTA keeps
//   QS      (16 KB, one stage)  its 64 query rows of Q_m, both column blocks: the S^T B operand
//   QK      (16 KB, two stages) all 128 query rows of Q_m, column block r: the dK B operand
//   dO      (32 KB, one stage)  the same two pieces of dO_m for dV [0,16K) and dP^T [16K,32K)
//   KX, KY  (16 KB each)        column block r of K_n0 and of K_n1: the dQ B operand (one of
//                               them repeats this CTA's own K, which stays whole for S^T)
//   DSX, DSY (16 KB each)       dS^T of key tile n0 / n1 for this CTA's 64 query rows: the dQ
//                               A operand, written half by this CTA and half by the peer
// QS_m is free once S^T_m is computed, a whole query tile before S^T_{m+1} needs it again.
//
// Tensor memory (512 columns, per CTA): dK [0,128), dV [128,256), S^T / P^T [256,384),
// dP^T [384,512) with dS^T (bf16, packed two per column) over its first 64 columns and dQ over
// its last 64 (an M = 128 pair accumulator keeps its 64 rows in lanes 0..63 for columns 0..63
// of N and in lanes 64..127 for columns 64..127).
// Warps (384 threads per CTA): 0 TMA producer, 1 MMA issuer (rank 0) and tensor-memory owner,
// 4..7 P^T / dS^T (thread = key row), 8..11 dQ drain.  Barriers that the MMA issuer waits on live
// in rank 0 (TMA loads of both CTAs complete there; the warps of both CTAs arrive there); its
// commits arrive on the same barrier in both CTAs.
#pragma once

#include "fa_bwd.cuh"

namespace fa {

struct Bwd2Layout {
  static constexpr int D = 128;
  static constexpr int kBlock = 16384;  // 128 rows x 64 bf16 (one 128-byte-swizzled column block)
  static constexpr int kHalf = 8192;    // 64 rows x 64 bf16
  static constexpr int kK = 0;                    // own K, column blocks 0, 1 (S^T A operand)
  static constexpr int kV = kK + 2 * kBlock;      // own V (dP^T A operand)
  static constexpr int kKX = kV + 2 * kBlock;     // K of key tile n0, column block r (dQ B operand)
  static constexpr int kKY = kKX + kBlock;        // K of key tile n1, column block r
  static constexpr int kQS = kKY + kBlock;        // this CTA's 64 rows of Q, blocks 0, 1 (S^T B operand)
  static constexpr int kQK = kQS + kBlock;        // two stages: all rows of Q, block r (dK B operand)
  static constexpr int kdO = kQK + 2 * kBlock;    // [0,16K) all rows, block r (dV); [16K,32K) 64 rows, blocks 0, 1 (dP^T)
  static constexpr int kDSX = kdO + 2 * kBlock;   // dS^T of key tile n0, this CTA's 64 queries (dQ A operand)
  static constexpr int kDSY = kDSX + kBlock;      // dS^T of key tile n1
  static constexpr int kDQ = kDSY + kBlock;       // two 8 KB staging buffers: 64 rows x 32 fp32
  static constexpr int kLse = kDQ + 2 * 8192;     // two stages of 128 fp32 (-LSE2), with QK
  static constexpr int kDsum = kLse + 1024;       // two stages of 128 fp32 (-D), with QK
  static constexpr int kBar = kDsum + 1024;
  // kv_full, qs_full, qs_empty, q_full[2], q_empty[2], do_full, do_empty, s_full, dp_full, p_full,
  // dst_full, dss_full, ds_empty, dq_full, dq_free, acc_full, drain, lse_full[2], exit
  static constexpr int kNumBars = 22;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;  // the dynamic shared memory base is 1024-byte aligned
  static constexpr uint32_t kColDK = 0, kColDV = 128, kColS = 256, kColDP = 384, kColDQ = 448;
};
static_assert(Bwd2Layout::kBytes <= 227 * 1024, "shared memory per CTA");

// 16-byte store into the shared memory of a CTA of this cluster (shared::cluster address).
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
// Orders this thread's generic-proxy writes to shared memory anywhere in the cluster before later
// async-proxy (UMMA) reads.
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

template <bool CAUSAL>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(384, 1)
    bwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmQ64,
                const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                const __grid_constant__ CUtensorMap tmdO, const __grid_constant__ CUtensorMap tmdO64,
                const __grid_constant__ CUtensorMap tmdQacc64, const BwdParams prm) {
  using L = Bwd2Layout;
  constexpr int D = L::D;

  extern __shared__ __align__(1024) uint8_t smem[];
  // identical in both CTAs of the pair, so both leave before any pair operation
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(prm.status, 0, kSiteBwd | 0x7E);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t *kv_full = bars + 0, *qs_full = bars + 1, *qs_empty = bars + 2, *q_full = bars + 3;
  uint64_t *q_empty = bars + 5, *do_full = bars + 7, *do_empty = bars + 8, *s_full = bars + 9;
  uint64_t *dp_full = bars + 10, *p_full = bars + 11, *dst_full = bars + 12, *dss_full = bars + 13;
  uint64_t *ds_empty = bars + 14, *dq_full = bars + 15, *dq_free = bars + 16, *acc_full = bars + 17;
  uint64_t *drain = bars + 18, *lse_full = bars + 19, *exit_bar = bars + 21;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kMisc + 4);

  const uint32_t rank = cluster_rank();
  const int r = static_cast<int>(rank);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_units = (prm.n_kv_tiles + 1) / 2;
  int bh, u;  // key-tile pair u = 0 (the most causal work) first, a few heads at a time
  cta_order(blockIdx.x >> 1, prm.BHkv, n_units, cta_head_group(prm.BHkv, n_units, CAUSAL), bh, u);
  const int n0 = 2 * u, n = n0 + r;                  // this CTA's key tile (n1 may lie past the end)
  const int m_begin = CAUSAL ? n0 : 0;               // first query tile that sees key tile n0
  const int n_it = prm.n_q_tiles - m_begin;          // >= 1

  if (threadIdx.x == 0) {
    mbar_init(kv_full, 1);
    mbar_init(qs_full, 1);
    mbar_init(qs_empty, 1);
    for (int st = 0; st < 2; ++st) {
      mbar_init(&q_full[st], 1);
      mbar_init(&q_empty[st], 1);
      mbar_init(&lse_full[st], 1);
    }
    mbar_init(do_full, 1);
    mbar_init(do_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    mbar_init(p_full, 8);    // one arrival per P / dS warp of either CTA
    mbar_init(dst_full, 8);
    mbar_init(dss_full, 8);
    mbar_init(ds_empty, 1);
    mbar_init(dq_full, 1);
    mbar_init(dq_free, 8);   // one arrival per drain warp of either CTA
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    mbar_init(exit_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised before any cross-CTA arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const Guard g{abort_flag, prm.status};

  if (warp < 4) {
    regs_to<kBwdRegsCtl, kBwdLaunchRegs>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer (both CTAs)
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmQ64);
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        prefetch_tmap(&tmdO);
        prefetch_tmap(&tmdO64);
        // rank 0's barriers, as shared::cluster addresses
        const uint32_t kv_full0 = peer_smem(smem_u32(kv_full), 0), do_full0 = peer_smem(smem_u32(do_full), 0);
        const uint32_t qs_full0 = peer_smem(smem_u32(qs_full), 0);
        if (r == 0) mbar_expect_tx(kv_full, 2 * 6 * L::kBlock);
        for (int b = 0; b < 2; ++b) {
          tma_load_3d_pair(smem + L::kK + b * L::kBlock, &tmK, 64 * b, n * kTile, bh, kv_full0);
          tma_load_3d_pair(smem + L::kV + b * L::kBlock, &tmV, 64 * b, n * kTile, bh, kv_full0);
        }
        tma_load_3d_pair(smem + L::kKX, &tmK, 64 * r, n0 * kTile, bh, kv_full0);
        tma_load_3d_pair(smem + L::kKY, &tmK, 64 * r, (n0 + 1) * kTile, bh, kv_full0);
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
          const int m = m_begin + it, st = it & 1;
          const int y64 = m * kTile + 64 * r;  // this CTA's 64 query rows
          // QS_m (one stage: free once S^T_{m-1} is computed)
          if (!(ok = wait(qs_empty, (it & 1) ^ 1, g, kSiteBwd | 0x30))) break;
          if (r == 0) mbar_expect_tx(qs_full, 2 * L::kBlock);
          tma_load_3d_pair(smem + L::kQS, &tmQ64, 0, y64, bh, qs_full0);
          tma_load_3d_pair(smem + L::kQS + L::kHalf, &tmQ64, 64, y64, bh, qs_full0);
          // QK_m with -LSE2_m, -D_m (two stages: free once dK_{m-2} is computed)
          if (!(ok = wait(&q_empty[st], ((it >> 1) & 1) ^ 1, g, kSiteBwd | 0x31))) break;
          if (r == 0) mbar_expect_tx(&q_full[st], 2 * L::kBlock);
          tma_load_3d_pair(smem + L::kQK + st * L::kBlock, &tmQ, 64 * r, m * kTile, bh,
                           peer_smem(smem_u32(&q_full[st]), 0));
          mbar_expect_tx(&lse_full[st], 1024);
          const size_t off = static_cast<size_t>(bh) * prm.Npad + static_cast<size_t>(m) * kTile;
          bulk_load(smem + L::kLse + 512 * st, prm.nlse2 + off, 512, &lse_full[st]);
          bulk_load(smem + L::kDsum + 512 * st, prm.ndsum + off, 512, &lse_full[st]);
          // dO_m (one stage: free once dV_{m-1} is computed)
          if (!(ok = wait(do_empty, (it & 1) ^ 1, g, kSiteBwd | 0x32))) break;
          if (r == 0) mbar_expect_tx(do_full, 2 * 2 * L::kBlock);
          tma_load_3d_pair(smem + L::kdO, &tmdO, 64 * r, m * kTile, bh, do_full0);
          tma_load_3d_pair(smem + L::kdO + L::kBlock, &tmdO64, 0, y64, bh, do_full0);
          tma_load_3d_pair(smem + L::kdO + L::kBlock + L::kHalf, &tmdO64, 64, y64, bh, do_full0);
        }
        (void)ok;
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------------- MMA (rank 0)
      // Issue order per query tile m: dP_m, dV_m, S_{m+1}, dK_m, dQ_m.
      if (lane == 0 && r == 0) {
        constexpr uint32_t idKK = idesc_bf16_f32(256, 128, false, false);  // S^T, dP^T
        constexpr uint32_t idKM = idesc_bf16_f32(256, D, false, true);     // dV, dK: A in TMEM, B MN-major
        constexpr uint32_t idQ = idesc_bf16_f32(128, D, true, true);       // dQ: M = 128 over the pair
        // Descriptors: one base per operand buffer, opaque to the compiler inside each query tile
        // (so it neither hoists a descriptor per instruction nor recomputes them one by one); each
        // instruction adds its compile-time offset (bytes / 16) to the address field.
        const uint32_t s0 = smem_u32(smem);
        auto base = [&](uint32_t off, uint32_t lbo) {
          uint64_t d = sdesc_sw128(s0 + off, lbo, 1024);
          asm volatile("" : "+l"(d));
          return d;
        };
        // S^T or dP^T: A = own K or V (column block b at b * 16K), B = this CTA's 64 query rows
        // (column block b at b * 8K)
        auto issue_rows = [&](uint32_t d_col, uint64_t dA, uint64_t dB) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t b = kk >> 2, k16 = (kk & 3) * 32;
            mma_ss_pair(tmem + d_col, dA + ((b * L::kBlock + k16) >> 4), dB + ((b * L::kHalf + k16) >> 4), idKK,
                        kk > 0);
          }
        };
        bool ok = wait(kv_full, 0, g, kSiteBwd | 0x33) && wait(qs_full, 0, g, kSiteBwd | 0x34);
        if (ok) {
          tc_fence_after();
          issue_rows(L::kColS, base(L::kK, 16), base(L::kQS, 16));
          tc_commit_pair(s_full);
          tc_commit_pair(qs_empty);
        }
        for (int it = 0; ok && it < n_it; ++it) {
          const int st = it & 1;
          const uint32_t ph = it & 1;
          // dP^T = V dO^T (its last 64 columns hold dQ of the previous tile)
          if (!(ok = wait(do_full, ph, g, kSiteBwd | 0x35))) break;
          if (it > 0 && !(ok = wait_cluster(dq_free, ph ^ 1, g, kSiteBwd | 0x36))) break;
          tc_fence_after();
          issue_rows(L::kColDP, base(L::kV, 16), base(L::kdO + L::kBlock, 16));
          tc_commit_pair(dp_full);
          // dV += P^T dO (B: all query rows of column block r)
          if (!(ok = wait_cluster(p_full, ph, g, kSiteBwd | 0x37))) break;
          tc_fence_after();
          {
            const uint64_t dB = base(L::kdO, L::kBlock);
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_ts_pair(tmem + L::kColDV, tmem + L::kColS + 8 * kk, dB + ((kk * 2048) >> 4), idKM,
                          (it > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit_pair(do_empty);
          // S^T of the next query tile (P_m in the S columns has been read by the dV MMA above)
          if (it + 1 < n_it) {
            if (!(ok = wait(qs_full, (it + 1) & 1, g, kSiteBwd | 0x38))) break;
            tc_fence_after();
            issue_rows(L::kColS, base(L::kK, 16), base(L::kQS, 16));
            tc_commit_pair(s_full);
            tc_commit_pair(qs_empty);
          }
          // dK += dS^T Q
          if (!(ok = wait_cluster(dst_full, ph, g, kSiteBwd | 0x39))) break;
          if (!(ok = wait(&q_full[st], (it >> 1) & 1, g, kSiteBwd | 0x41))) break;
          tc_fence_after();
          {
            const uint64_t dB = base(L::kQK + st * L::kBlock, L::kBlock);
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              mma_ts_pair(tmem + L::kColDK, tmem + L::kColDP + 8 * kk, dB + ((kk * 2048) >> 4), idKM,
                          (it > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit_pair(&q_empty[st]);
          // dQ_m = dS K over both key tiles of the pair (K-dimension: the keys of n0, then of n1)
          if (!(ok = wait_cluster(dss_full, ph, g, kSiteBwd | 0x3A))) break;
          tc_fence_after();
          {
            const uint64_t dA = base(L::kDSX, L::kBlock), dB = base(L::kKX, L::kBlock);
#pragma unroll
            for (int kk = 0; kk < 2 * kTile / 16; ++kk) {
              const uint32_t off = (kk >> 3) * L::kBlock + (kk & 7) * 2048;  // DSY / KY follow DSX / KX
              mma_ss_pair(tmem + L::kColDQ, dA + (off >> 4), dB + (off >> 4), idQ, kk > 0);
            }
          }
          tc_commit_pair(dq_full);
          tc_commit_pair(ds_empty);
        }
        if (ok) tc_commit_pair(acc_full);
        tc_commit_pair_local(drain);
        drain_wait(drain, 0);
      }
    }
  } else if (warp < 8) {
    regs_to<kBwdRegsP, kBwdLaunchRegs>();
    // --------------------------------------------------- P^T and dS^T rows (both CTAs)
    const int quarter = warp & 3;
    const int j = quarter * 32 + lane;  // key row within this CTA's tile
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + L::kColS + lane_off, tdP = tmem + L::kColDP + lane_off;
    const uint32_t p_full0 = peer_smem(smem_u32(p_full), 0), dst_full0 = peer_smem(smem_u32(dst_full), 0);
    const uint32_t dss_full0 = peer_smem(smem_u32(dss_full), 0);
    // this CTA's dS^T slot (key tile n) here and in the peer: the peer's half of the queries goes there
    uint8_t* slot = smem + (r == 0 ? L::kDSX : L::kDSY);
    const uint32_t slot_peer = peer_smem(smem_u32(slot), rank ^ 1u);
    const float2 c2 = make_float2(prm.scale_log2, prm.scale_log2);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int m = m_begin + it, st = it & 1;
      const uint32_t ph = it & 1;
      const float4* nl4 = reinterpret_cast<const float4*>(smem + L::kLse + 512 * st);
      const float4* nd4 = reinterpret_cast<const float4*>(smem + L::kDsum + 512 * st);
      if (!(ok = wait_warp(&lse_full[st], (it >> 1) & 1, g, kSiteBwd | 0x3B))) break;
      if (!(ok = wait_warp(s_full, ph, g, kSiteBwd | 0x3C))) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sr[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(sr[c]);
      float p[kTile];
      // causal: query i of tile m does not see key j of tile n when n*128 + j > m*128 + i, i.e. i < thr
      const int thr = (n - m) * kTile + j;
      const bool diag = CAUSAL && n >= m;
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
            pv.x = exp2_sfu(x.x);
            pv.y = exp2_sfu(x.y);
            if (diag) {
              if (ii < thr) pv.x = 0.0f;
              if (ii + 1 < thr) pv.y = 0.0f;
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
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(p_full0);

      if (!(ok = wait_warp(dp_full, ph, g, kSiteBwd | 0x3D))) break;
      tc_fence_after();
      if (it > 0 && !(ok = wait_warp(ds_empty, ph ^ 1, g, kSiteBwd | 0x3E))) break;
      uint32_t dp_[2][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        if ((c & 1) == 0) {  // dP^T columns 64 at a time (all read before any dS^T lands on them)
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
        // dS^T to tensor memory for dK (over dP^T columns read above)
        tmem_st16(tdP + 16 * c, w);
        // queries 32c .. 32c+31 to the dS^T slot of key tile n: here when they are this CTA's
        // 64 dQ rows (half c >> 1 == r), else in the peer
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint32_t o = sw128_offset(j, (c & 1) * 32 + q4 * 8);
          const uint4 v = make_uint4(w[4 * q4], w[4 * q4 + 1], w[4 * q4 + 2], w[4 * q4 + 3]);
          if ((c >> 1) == r)
            *reinterpret_cast<uint4*>(slot + o) = v;
          else
            st_cluster_v4(slot_peer + o, v);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(dst_full0);
      // the slots were written through the generic proxy, here and in the peer: make them visible
      // to the UMMA reads, then release them at cluster scope
      fence_proxy_async_all();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(dss_full0);
    }
    if (ok) ok = wait_warp(acc_full, 0, g, kSiteBwd | 0x3F);
    if (ok) {
      tc_fence_after();
      const int key = n * kTile + j;
      const bool store = key < prm.Nk;
      const size_t rowoff = (static_cast<size_t>(bh) * prm.Nk + (store ? key : 0)) * D;
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const uint32_t tcol = tmem + (which == 0 ? L::kColDK : L::kColDV) + lane_off;
        const float mul = which == 0 ? prm.scale : 1.0f;
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
    // ---------------------------------------------------------- dQ drain (both CTAs)
    // This CTA's 64 query rows of dQ_m: lane l < 64 holds row l, columns 0..63 of d; lane l >= 64
    // row l - 64, columns 64..127.  They leave 32 columns at a time through two 8 KB staging
    // buffers (one per half of d) and TMA reduce-adds into the fp32 accumulator.
    const int quarter = warp & 3;
    const int lrow = quarter * 32 + lane;
    const int qrow = lrow & 63, dhalf = lrow >> 6;
    const bool leader = (warp == 8 && lane == 0);
    const uint32_t tdQ = tmem + L::kColDQ + (static_cast<uint32_t>(quarter * 32) << 16);
    const uint32_t dq_free0 = peer_smem(smem_u32(dq_free), 0);
    uint8_t* buf = smem + L::kDQ + dhalf * 8192;
    if (leader) prefetch_tmap(&tmdQacc64);
    bool ok = true;
    for (int it = 0; it < n_it; ++it) {
      const int m = m_begin + it;
      const bool okl = ok && wait_warp(dq_full, it & 1, g, kSiteBwd | 0x40);
      if (!(ok = group_and(1, 128, okl))) break;
      tc_fence_after();
      uint32_t a[2][32];
      tmem_ld32(tdQ, a[0]);
      tmem_ld32(tdQ + 32, a[1]);
      tmem_wait_ld();
      reg_fence(a[0]);
      reg_fence(a[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster_relaxed(dq_free0);  // the dQ columns may be overwritten now
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (leader) bulk_wait_read<0>();  // the reduces that last used the buffers have read them
        named_barrier(1, 128);
#pragma unroll
        for (int v = 0; v < 8; ++v)
          *reinterpret_cast<uint4*>(buf + qrow * 128 + (((v ^ qrow) & 7) << 4)) =
              make_uint4(a[h][4 * v], a[h][4 * v + 1], a[h][4 * v + 2], a[h][4 * v + 3]);
        fence_proxy_async();
        named_barrier(1, 128);
        if (leader) {
          const int y = m * kTile + 64 * r;
          tma_reduce_add_3d(&tmdQacc64, 32 * h, y, bh, smem + L::kDQ);
          tma_reduce_add_3d(&tmdQacc64, 64 + 32 * h, y, bh, smem + L::kDQ + 8192);
          bulk_commit();
        }
      }
    }
    if (leader) bulk_wait<0>();
  }

  // Pair teardown: each CTA tells the other it is done (bounded), then both release tensor memory.
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) mbar_arrive_cluster(peer_smem(smem_u32(exit_bar), rank ^ 1u));
  if (warp == 1) {
    drain_wait(exit_bar, 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace fa
