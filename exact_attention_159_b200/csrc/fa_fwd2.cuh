// fa_fwd2.cuh -- forward exact attention on a cluster pair of SMs (2-CTA UMMA), d = 128.
//
// The FlashAttention-4 pages describe CTA pairs that share one large tile, each
// carrying half of the load and exchanging operands without a trip to HBM
// ("C. Le Duo de Cuisiniers (2-CTA)").  Here a cluster of two CTAs computes
// every S = Q K^T and O += P V with one tcgen05.mma.cta_group::2 of M = 256:
// the A rows (Q, or P from tensor memory) come 128 from each CTA, and the B
// operand is split by N between the two CTAs' shared memory -- each CTA loads
// only 64 of the 128 keys of a K tile and 64 of the 128 columns of a V tile,
// halving the K/V TMA traffic and the shared-memory operand reads per SM (the
// limit of the single-CTA kernel).
//
// A cluster owns four consecutive 128-row query tiles 4u .. 4u+3 of one head:
// slot t (ping-pong, 0 or 1) pairs tile 4u+2t (CTA rank 0) with 4u+2t+1
// (rank 1).  Both CTAs of a slot step through the same key tiles; under the
// causal mask rank 0 sees one key tile beyond its diagonal, fully masked.
// Warp roles per CTA (640 threads) as in the single-CTA kernel: warp 0 TMA,
// warp 1 MMA (rank 0 issues for the pair; both ranks allocate tensor memory
// together), warps 4..19 softmax with every row split over two threads.
// Synchronisation across the pair:
//   * both CTAs' TMA loads complete on rank 0's q_full / k_full / v_full;
//   * rank 0's commits arrive on s_full / o_full / kv_empty in both CTAs;
//   * each softmax warp of either CTA arrives once on rank 0's p_full;
//   * a bounded remote-arrive handshake precedes the release of tensor memory.
#pragma once

#include "fa_fwd.cuh"

namespace fa {

struct Fwd2Layout {
  static constexpr int D = 128;
  static constexpr int kQBytes = kTile * D * 2;       // one 128 x 128 query tile
  static constexpr int kKHalf = 64 * D * 2;           // 64 keys x 128 columns
  static constexpr int kVHalf = kTile * 64 * 2;       // 128 keys x 64 columns
  static constexpr int kStages = 4;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 2 * kQBytes;
  static constexpr int kV = kK + kStages * kKHalf;
  static constexpr int kBar = kV + kStages * kVHalf;
  // q_full, k_full[S], v_full[S], kv_empty[S], s_full[2], p_full[2], o_full[2], drain, exit
  static constexpr int kNumBars = 1 + 3 * kStages + 8;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kXchg = kMisc + 16;
  static constexpr int kBytes = kXchg + 2 * 2 * 128 * 4;
  static constexpr int kThreads = 640;
};

struct Fwd2Params {
  __nv_bfloat16* O;
  float* LSE;
  int N, BH, n_quads;  // n_quads = ceil(ceil(N / 128) / 4): clusters per head
  float scale_log2, tau;
  int* status;
};

// Register split (setmaxnreg) of the pair kernel: 128 * 56 + 512 * 104 <= 640 * 96, the launch's total.
constexpr int kFwd2RegsCtl = 56, kFwd2RegsSoftmax = 104;
static_assert(128 * kFwd2RegsCtl + 512 * kFwd2RegsSoftmax <= 640 * ((65536 / 640) / 8 * 8),
              "pair forward register split exceeds the launch's");

template <bool CAUSAL, int POLY16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(640, 1)
    fwd2_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK64,
                const __grid_constant__ CUtensorMap tmV, const Fwd2Params prm) {
  using L = Fwd2Layout;
  constexpr int D = L::D;
  constexpr int S = L::kStages;

  extern __shared__ __align__(1024) uint8_t smem[];
  // identical in both CTAs of the pair, so both leave before any pair operation
  if ((smem_u32(smem) & 1023u) != 0) {
    if (threadIdx.x == 0) atomicCAS(prm.status, 0, kSiteFwd | 0x7E);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + S;
  uint64_t* kv_empty = v_full + S;
  uint64_t* s_full = kv_empty + S;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 2;
  uint64_t* exit_bar = drain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kMisc + 4);

  const uint32_t rank = cluster_rank();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bh, unit;
  cta_order(blockIdx.x >> 1, prm.BH, prm.n_quads, cta_head_group(prm.BH, prm.n_quads, CAUSAL), bh, unit);
  const int quad = prm.n_quads - 1 - unit;  // heaviest causal work first
  const int n_tiles = (prm.N + kTile - 1) / kTile;
  int nkv[2];
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int first = 4 * quad + 2 * t;  // rank 0's tile of slot t
    nkv[t] = first < n_tiles ? (CAUSAL ? min(first + 2, n_tiles) : n_tiles) : 0;
  }
  const int nkv_max = nkv[0] > nkv[1] ? nkv[0] : nkv[1];

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 16);  // one arrival per softmax warp of the slot, both CTAs
      mbar_init(&o_full[t], 1);
    }
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
    regs_to<kFwd2RegsCtl, (65536 / L::kThreads) / 8 * 8>();
    if (warp == 0) {
      // ---------------------------------------------------------- producer
      if (lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmK64);
        prefetch_tmap(&tmV);
        const uint32_t q_full0 = peer_smem(smem_u32(q_full), 0);
        if (rank == 0) mbar_expect_tx(q_full, ((nkv[0] > 0) + (nkv[1] > 0)) * 2 * L::kQBytes);
        for (int t = 0; t < 2; ++t)
          if (nkv[t] > 0)
            for (int c = 0; c < 2; ++c)
              tma_load_3d_pair(smem + L::kQ + t * L::kQBytes + c * 16384, &tmQ, 64 * c,
                               (4 * quad + 2 * t + rank) * kTile, bh, q_full0);
        bool ok = true;
        for (int j = 0; j < nkv_max; ++j) {
          const int s = j % S;
          if (!(ok = wait(&kv_empty[s], ((j / S) & 1) ^ 1, g, kSiteFwd | 0x21))) break;
          if (rank == 0) {
            mbar_expect_tx(&k_full[s], 2 * L::kKHalf);
            mbar_expect_tx(&v_full[s], 2 * L::kVHalf);
          }
          // K: keys 64*rank .. +63 of the tile, both 64-column chunks; V: all 128 keys, columns 64*rank ..
          for (int c = 0; c < 2; ++c)
            tma_load_3d_pair(smem + L::kK + s * L::kKHalf + c * 8192, &tmK64, 64 * c, j * kTile + 64 * rank, bh,
                             peer_smem(smem_u32(&k_full[s]), 0));
          tma_load_3d_pair(smem + L::kV + s * L::kVHalf, &tmV, 64 * rank, j * kTile, bh,
                           peer_smem(smem_u32(&v_full[s]), 0));
        }
        (void)ok;
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------------- MMA
      if (lane == 0 && rank == 0) {
        constexpr uint32_t idS = idesc_bf16_f32(256, 128, false, false);  // Q (K-major) x K half (K-major)
        constexpr uint32_t idO = idesc_bf16_f32(256, D, false, true);     // P (TMEM) x V half (MN-major)
        const uint32_t sQ = smem_u32(smem + L::kQ), sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
        auto issue_s = [&](int t, int s) {
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t offq = (kk >> 2) * 16384 + (kk & 3) * 32, offk = (kk >> 2) * 8192 + (kk & 3) * 32;
            mma_ss_pair(tmem + 128 * t, sdesc_sw128(sQ + t * L::kQBytes + offq, 16, 1024),
                        sdesc_sw128(sK + s * L::kKHalf + offk, 16, 1024), idS, kk > 0);
          }
        };
        auto issue_pv = [&](int t, int s, bool acc) {
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts_pair(tmem + 256 + D * t, tmem + 128 * t + 8 * kk,
                        sdesc_sw128(sV + s * L::kVHalf + kk * 2048, 16384, 1024), idO, (acc || kk > 0) ? 1u : 0u);
        };
        bool ok = wait(q_full, 0, g, kSiteFwd | 0x22) && wait(&k_full[0], 0, g, kSiteFwd | 0x23);
        if (ok) {
          tc_fence_after();
          for (int t = 0; t < 2; ++t)
            if (nkv[t] > 0) {
              issue_s(t, 0);
              tc_commit_pair(&s_full[t]);
            }
        }
        for (int j = 0; ok && j < nkv_max; ++j) {
          const int s = j % S;
          if (!(ok = wait(&v_full[s], (j / S) & 1, g, kSiteFwd | 0x24))) break;
          for (int t = 0; t < 2 && ok; ++t) {
            if (j >= nkv[t]) continue;
            if (!(ok = wait_cluster(&p_full[t], j & 1, g, kSiteFwd | 0x25))) break;
            tc_fence_after();
            issue_pv(t, s, j > 0);
            tc_commit_pair(&o_full[t]);
            if (j + 1 < nkv[t]) {
              const int s1 = (j + 1) % S;
              if (!(ok = wait(&k_full[s1], ((j + 1) / S) & 1, g, kSiteFwd | 0x26))) break;
              tc_fence_after();
              issue_s(t, s1);
              tc_commit_pair(&s_full[t]);
            }
          }
          // release the stage only if a later key tile will be loaded into it
          if (ok && j + S < nkv_max) tc_commit_pair(&kv_empty[s]);
        }
        tc_commit_pair_local(drain);
        drain_wait(drain, 0);
      }
    }
  } else {
    regs_to<kFwd2RegsSoftmax, (65536 / L::kThreads) / 8 * 8>();
    // ------------------------------------------- softmax / correction / epilogue
    const int t = (warp - 4) >> 3;
    const int h = ((warp - 4) >> 2) & 1;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + 128 * t + lane_off;
    const uint32_t tO = tmem + 256 + D * t + (D / 2) * h + lane_off;
    float* xchg = reinterpret_cast<float*>(smem + L::kXchg) + t * 256;
    const int bar_id = 1 + 4 * t + quarter;                            // the two warps sharing these rows
    const uint32_t p_full0 = peer_smem(smem_u32(&p_full[t]), 0);
    const int qt = 4 * quad + 2 * t + static_cast<int>(rank);
    const int row = qt * kTile + r;
    const float sl2 = prm.scale_log2;
    float m_ref = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv[t]; ++j) {
      // every exit decision is taken jointly by the two warps of a row (group_and), so neither is
      // ever left waiting at a barrier the other skipped; after a failed wait the block below
      // only reads stale TMEM columns of this CTA's own allocation before the joint exit
      const bool okl = ok && wait_warp(&s_full[t], j & 1, g, kSiteFwd | 0x27);
      tc_fence_after();
      uint32_t sr[2][32];
      tmem_ld32(tS + 64 * h, sr[0]);
      tmem_ld32(tS + 64 * h + 32, sr[1]);
      tmem_wait_ld();
      reg_fence(sr[0]);
      reg_fence(sr[1]);
#define S(c) __uint_as_float(sr[(c) >> 5][(c) & 31])
      const bool edge = (CAUSAL && j >= qt) || ((j + 1) * kTile > prm.N);
      if (edge) {
        const int key0 = j * kTile + 64 * h;
#pragma unroll
        for (int c = 0; c < 64; ++c) {
          const int key = key0 + c;
          if (key >= prm.N || (CAUSAL && key > row)) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
        }
      }
      float mx[2] = {S(0), S(32)};
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int c = 32 * q + 1; c < 32 * q + 31; c += 2) mx[q] = fmax3(mx[q], S(c), S(c + 1));
#pragma unroll
      for (int q = 0; q < 2; ++q) mx[q] = fmaxf(mx[q], S(32 * q + 31));
      const float mine = fmaxf(mx[0], mx[1]);
      xchg[128 * h + r] = mine;
      if (!(ok = group_and(bar_id, 64, okl))) break;
      const float m_new = fmaxf(m_ref, fmaxf(mine, xchg[128 * (h ^ 1) + r]) * sl2);
      const bool need = m_new > m_ref + prm.tau;
      const float alpha = need ? exp2_sfu(m_ref - m_new) : 1.0f;
      if (need) {
        l *= alpha;
        m_ref = m_new;
      }
      // a row with every key of this tile masked (rank 0 past its diagonal) keeps m_ref = -inf
      // only if it never saw a key; its P is 0 either way
      const float2 c2 = make_float2(sl2, sl2), nm2 = make_float2(-m_ref, -m_ref);
      float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = 32 * cc + 2 * e;
          const float2 x = __ffma2_rn(make_float2(S(c), S(c + 1)), c2, nm2);
          float2 p;
          if (!edge && POLY16 > 0 && e % (POLY16 > 0 ? 16 / POLY16 : 16) == 0) {
            p = exp2_poly2(x);
          } else {
            p.x = exp2_sfu(x.x);
            p.y = exp2_sfu(x.y);
          }
          if (e & 1)
            ls1 = __fadd2_rn(ls1, p);
          else
            ls0 = __fadd2_rn(ls0, p);
          pk[e] = pack_bf16x2(p.x, p.y);
        }
        tmem_st16(tS + 32 * h + 16 * cc, pk);
      }
#undef S
      const float2 ls = __fadd2_rn(ls0, ls1);
      l += ls.x + ls.y;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        ok = wait_warp(&o_full[t], (j - 1) & 1, g, kSiteFwd | 0x28);
        tc_fence_after();  // a failed wait is carried to the next joint decision
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + 32 * c, o);
          tmem_wait_ld();
          reg_fence(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(tO + 32 * c, o);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      // P and the corrected O are tensor memory, complete after tcgen05.wait::st: a relaxed arrival
      if (ok && lane == 0) mbar_arrive_cluster_relaxed(p_full0);
    }
    if (nkv[t] > 0) {
      // full row sum from the two halves (joint decision, as in the loop)
      const bool okl = ok && wait_warp(&o_full[t], (nkv[t] - 1) & 1, g, kSiteFwd | 0x29);
      if (okl) {
        tc_fence_after();
        xchg[128 * h + r] = l;
      }
      ok = group_and(bar_id, 64, okl);
    }
    if (ok && nkv[t] > 0) {
      const float l_row = l + xchg[128 * (h ^ 1) + r];
      const float inv_l = 1.0f / l_row;
      const bool store = row < prm.N;
      __nv_bfloat16* orow = prm.O + (static_cast<size_t>(bh) * prm.N + (store ? row : 0)) * D + (D / 2) * h;
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
        reg_fence(o);
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        }
      }
      if (store && h == 0)
        prm.LSE[static_cast<size_t>(bh) * prm.N + row] = (m_ref + log2f(l_row)) * 0.69314718055994531f;
    }
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
