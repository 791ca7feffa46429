// fa_fwd.cuh -- forward exact attention on sm_100a (tcgen05 + TMEM + TMA).
//
// One CTA owns two 128-row query tiles of one (batch, head) ("ping-pong":
// FlashAttention-4 pages, "A. La Danse du Ping-Pong" -- while the tensor core
// works for one tile, the softmax warps work on the other).  Warp roles
// ("The Technical Edge": warp specialisation into load / MMA / softmax /
// output stages):
//   warp 0        TMA producer: Q tiles once, then a ring of K/V tiles
//   warp 1        MMA issuer (one thread) and TMEM owner
//   warps 2, 3    idle (they complete the first warpgroup)
//   warps 4..7    softmax + correction + epilogue for query tile 0
//   warps 8..11   the same for query tile 1
// One thread owns one score row: it loads all 128 scores of its row for a key
// tile into registers, so the row maximum and the row sum need no exchange
// between threads, and its 128 independent exponentials give the instruction-
// level parallelism that lets a share of them run as the cubic on the FMA
// pipe alongside the SFU.  Registers are re-split per warpgroup with
// setmaxnreg (56 for the control warps, 224 for the softmax warps, of the
// 168 x 384 launched).  The softmax arithmetic uses packed fp32x2 FMA/add.
// Tensor memory (512 columns x 128 lanes x 32 bit, "TMEM (256 KB per SM)"):
//   S_t = Q_t K^T  fp32, 128 columns at 128*t; P_t (bf16, packed two per
//   column) is written back over the first 64 columns of S_t and read from
//   there by the P.V MMA; O_t fp32, D columns at 256 + D*t.
// Online softmax in base 2 with the running row maximum m (log2 units) and
// conditional rescaling (ainvest page, "The Technical Edge": the running
// output is rescaled only when the row maximum has moved by a large amount):
// O and l are rescaled only when the
// tile maximum exceeds the reference maximum by more than tau = 8; otherwise
// the stale reference is kept, so P <= 2^8.  The result is exact either way
// because O / l and LSE use the same reference.
// A fixed share (POLY16 / 16) of the exponentials of interior tiles runs as the cubic
// polynomial on the FMA pipe, the rest on the SFU (same section: a cubic on
// the CUDA cores takes load off the special-function units).
#pragma once

#include <type_traits>

#include "exp2_poly.cuh"
#include "sm100.cuh"

namespace fa {

constexpr int kTile = 128;          // rows of a Q or K/V tile
constexpr float kRescaleTau = 8.0f;  // log2 units

// Error sites reported through the status word (low byte = kernel, next = site).
enum : int { kSiteFwd = 0x100, kSiteBwd = 0x200 };

struct FwdParams {
  __nv_bfloat16* O;   // [BH, N, D]
  float* LSE;         // [BH, N], natural log
  float* O_acc;       // [BH, N, D] fp32: when set, this call's (O, LSE) is folded into (O_acc, LSE_acc)
  float* LSE_acc;     // [BH, N]       by their log-sum-exp instead of being written to O, LSE
  int acc_first;      // 1: the accumulators are initialised from this call
  int N;              // query rows per head
  int Nk;             // key rows per head
  int BH;             // batch * query heads
  int Hq, G;          // query heads per batch entry; query heads per key/value head
  int off;            // Nk - N: query row i sees keys j <= i + off when causal
  int n_pairs;        // ceil(ceil(N / 128) / 2)
  float scale_log2;   // softmax scale * log2(e)
  float tau;          // rescale threshold (log2 units)
  int* status;
};

template <int D>
struct FwdLayout {
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kStages = D == 128 ? 2 : 3;
  static constexpr int kQ = 0;
  static constexpr int kK = kQ + 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kBar = kV + kStages * kTileBytes;
  // q, k_full[S], v_full[S], k_empty[S], v_empty[S], s_full[2], p_full[2], o_full[2], drain
  static constexpr int kNumBars = 1 + 4 * kStages + 7;
  static constexpr int kMisc = kBar + kNumBars * 8;
  static constexpr int kBytes = kMisc + 16;  // the dynamic shared memory base is 1024-byte aligned
  static constexpr int kThreads = 384;
  static constexpr int kLaunchRegs = (65536 / kThreads) / 8 * 8;  // per-thread registers at launch
};

// Bounded wait that ignores the abort flag (used only to drain in-flight async work).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer() - t0 > 200000000ull) break;
  }
}

// Register split (setmaxnreg): 128 * 56 + 256 * 224 = 384 * 168, the launch's total.  Each
// setmaxnreg heads its role's branch so the register budget of that code is unambiguous.
constexpr int kFwdRegsCtl = 56, kFwdRegsSoftmax = 224;
static_assert(128 * kFwdRegsCtl + 256 * kFwdRegsSoftmax <= 384 * ((65536 / 384) / 8 * 8),
              "forward register split exceeds the launch's");

// GEN: grouped-query heads and / or N != Nk; without it (one query head per key/value head,
// N == Nk) the group and offset terms are compile-time constants.
template <int D, bool CAUSAL, int POLY16, bool GEN>
__global__ void __launch_bounds__(384, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const FwdParams prm) {
  using L = FwdLayout<D>;
  constexpr int S = L::kStages;
  constexpr int T = L::kTileBytes;
  constexpr int kChunks = D / 64;  // 128-byte swizzle chunks of 64 bf16 along d

  extern __shared__ __align__(1024) uint8_t smem[];
  if ((smem_u32(smem) & 1023u) != 0) {  // swizzled tiles need a 1024-byte aligned base
    if (threadIdx.x == 0) atomicCAS(prm.status, 0, kSiteFwd | 0x7F);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* bar_q = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + S;
  uint64_t* k_empty = v_full + S;  // K and V stages are released separately: K(j) is done
  uint64_t* v_empty = k_empty + S;  // once both S(t, j) are, about an iteration before V(j)
  uint64_t* s_full = v_empty + S;
  uint64_t* p_full = s_full + 2;
  uint64_t* o_full = p_full + 2;
  uint64_t* drain = o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  int* abort_flag = reinterpret_cast<int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int bh, unit;  // heaviest causal work (the last query tiles) first, a few heads at a time
  cta_order(blockIdx.x, prm.BH, prm.n_pairs, cta_head_group(prm.BH, prm.n_pairs, CAUSAL), bh, unit);
  const int pair = prm.n_pairs - 1 - unit;
  const int Nk = GEN ? prm.Nk : prm.N;
  const int off = GEN ? prm.off : 0;
  const int n_tiles = (prm.N + kTile - 1) / kTile;     // query tiles
  const int n_kv = (Nk + kTile - 1) / kTile;           // key / value tiles
  // key / value head of this query head (grouped-query attention: G query heads share one)
  const int bkv = GEN ? (bh / prm.Hq) * (prm.Hq / prm.G) + (bh % prm.Hq) / prm.G : bh;
  int nkv[2];  // key tiles query tile qt sees: those holding a key <= its last row + off
#pragma unroll
  for (int t = 0; t < 2; ++t) {
    const int qt = 2 * pair + t;
    const int last_key = qt * kTile + kTile - 1 + off;
    nkv[t] = qt >= n_tiles ? 0 : !CAUSAL ? n_kv : last_key < 0 ? 0 : min(last_key / kTile + 1, n_kv);
  }
  const int nkv_max = nkv[0] > nkv[1] ? nkv[0] : nkv[1];

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int s = 0; s < S; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_full[t], 1);
    }
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
    regs_to<kFwdRegsCtl, L::kLaunchRegs>();
    if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && nkv_max > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_expect_tx(bar_q, ((nkv[0] > 0) + (nkv[1] > 0)) * T);
      for (int t = 0; t < 2; ++t)
        if (nkv[t] > 0)
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(smem + L::kQ + t * T + c * 16384, &tmQ, 64 * c, (2 * pair + t) * kTile, bh, bar_q);
      // K(j) then V(j): the order in which their stages are released
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      for (int j = 0; j < nkv_max; ++j) {
        const int s = j % S;
        const uint32_t ph = (j / S) & 1;
        if (!(ok = wait(&k_empty[s], ph ^ 1, g, kSiteFwd | 1))) break;
        mbar_expect_tx(&k_full[s], T);
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d(smem + L::kK + s * T + c * 16384, &tmK, 64 * c, j * kTile, bkv, &k_full[s]);
        ++k_issued;
        if (!(ok = wait(&v_empty[s], ph ^ 1, g, kSiteFwd | 12))) break;
        mbar_expect_tx(&v_full[s], T);
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d(smem + L::kV + s * T + c * 16384, &tmV, 64 * c, j * kTile, bkv, &v_full[s]);
        ++v_issued;
      }
      if (!ok) {  // let copies already in flight land before the CTA exits
        drain_wait(bar_q, 0);
        for (int i = k_issued - S > 0 ? k_issued - S : 0; i < k_issued; ++i) drain_wait(&k_full[i % S], (i / S) & 1);
        for (int i = v_issued - S > 0 ? v_issued - S : 0; i < v_issued; ++i) drain_wait(&v_full[i % S], (i / S) & 1);
      }
    }
    } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    // One thread issues every UMMA, per key tile j in the order P.V(0, j), S(0, j+1), P.V(1, j),
    // S(1, j+1): the order is what keeps the two tiles' softmax phases half a period apart.  The
    // tensor pipe takes only about one instruction ahead of its issuing thread, so the barrier
    // waits between batches cost pipe time (80-90 clocks per 64-clock UMMA here, with the softmax
    // warps busy on the same SM); every way of sharing the issue between two threads was slower.
    if (lane == 0 && nkv_max > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(128, 128, false, false);  // Q (K-major) x K (K-major)
      constexpr uint32_t idO = idesc_bf16_f32(128, D, false, true);     // P (TMEM) x V (MN-major)
      const uint32_t sQ = smem_u32(smem + L::kQ), sK = smem_u32(smem + L::kK), sV = smem_u32(smem + L::kV);
      auto issue_s = [&](int t, int s) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
          mma_ss(tmem + 128 * t, sdesc_sw128(sQ + t * T + off, 16, 1024), sdesc_sw128(sK + s * T + off, 16, 1024),
                 idS, kk > 0);
        }
      };
      auto issue_pv = [&](int t, int s, bool acc) {
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk)
          mma_ts(tmem + 256 + D * t, tmem + 128 * t + 8 * kk, sdesc_sw128(sV + s * T + kk * 2048, 16384, 1024), idO,
                 (acc || kk > 0) ? 1u : 0u);
      };
      bool ok = wait(bar_q, 0, g, kSiteFwd | 2) && wait(&k_full[0], 0, g, kSiteFwd | 3);
      if (ok) {
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (nkv[t] > 0) {
            issue_s(t, 0);
            tc_commit(&s_full[t]);
          }
        tc_commit(&k_empty[0]);  // K(0) is free once both S(t, 0) are done
      }
      for (int j = 0; ok && j < nkv_max; ++j) {
        const int s = j % S;
        if (!(ok = wait(&v_full[s], (j / S) & 1, g, kSiteFwd | 4))) break;
        for (int t = 0; t < 2 && ok; ++t) {
          if (j >= nkv[t]) continue;
          if (!(ok = wait(&p_full[t], j & 1, g, kSiteFwd | 5))) break;
          tc_fence_after();
          issue_pv(t, s, j > 0);
          tc_commit(&o_full[t]);
          if (j + 1 < nkv[t]) {
            const int s1 = (j + 1) % S;
            if (!(ok = wait(&k_full[s1], ((j + 1) / S) & 1, g, kSiteFwd | 6))) break;
            tc_fence_after();
            issue_s(t, s1);
            tc_commit(&s_full[t]);
          }
        }
        if (ok) {
          tc_commit(&v_empty[s]);                                 // V(j): both P.V issued
          if (j + 1 < nkv_max) tc_commit(&k_empty[(j + 1) % S]);  // K(j+1): both S(t, j+1) issued
        }
      }
      tc_commit(drain);
      drain_wait(drain, 0);
    }
    }
  } else {
    regs_to<kFwdRegsSoftmax, L::kLaunchRegs>();
    // ------------------------------------------- softmax / correction / epilogue
    // One thread per score row: warps 4..7 hold the 128 rows of query tile 0 (one TMEM lane
    // quarter each), warps 8..11 those of tile 1.  A thread keeps its whole row of 128 scores in
    // registers, so the row maximum needs no exchange with another thread.
    const int t = (warp - 4) >> 2;   // query tile
    const int quarter = warp & 3;    // TMEM lanes this warp may touch: 32*quarter .. +31
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tS = tmem + 128 * t + lane_off;
    const uint32_t tO = tmem + 256 + D * t + lane_off;
    const int qt = 2 * pair + t;
    const int row = qt * kTile + r;  // query row within the head
    const float sl2 = prm.scale_log2;
    float m_ref = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < nkv[t]; ++j) {
      if (!(ok = wait_warp(&s_full[t], j & 1, g, kSiteFwd | 7))) break;
      tc_fence_after();
      uint32_t sr[4][32];
#pragma unroll
      for (int c = 0; c < 4; ++c) tmem_ld32(tS + 32 * c, sr[c]);
      tmem_wait_ld();
#pragma unroll
      for (int c = 0; c < 4; ++c) reg_fence(sr[c]);
      // scores stay in the registers tcgen05.ld wrote (S(c) reads key column c as fp32)
#define S(c) __uint_as_float(sr[(c) >> 5][(c) & 31])
      // masking: keys past the end, and (causal) keys beyond the first row's reach
      const bool edge = (CAUSAL && j * kTile + kTile - 1 > qt * kTile + off) || ((j + 1) * kTile > Nk);
      if (edge) {
#pragma unroll
        for (int c = 0; c < kTile; ++c) {
          const int key = j * kTile + c;
          if (key >= Nk || (CAUSAL && key > row + off)) sr[c >> 5][c & 31] = __float_as_uint(-INFINITY);
        }
      }
      // row maximum: four chains of 3-input max
      float mx[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        mx[q] = S(32 * q);
#pragma unroll
        for (int c = 32 * q + 1; c < 32 * q + 31; c += 2) mx[q] = fmax3(mx[q], S(c), S(c + 1));
        mx[q] = fmaxf(mx[q], S(32 * q + 31));
      }
      const float m_new = fmaxf(m_ref, fmax3(mx[0], mx[1], fmaxf(mx[2], mx[3])) * sl2);
      const bool need = m_new > m_ref + prm.tau;
      const float alpha = need ? exp2_sfu(m_ref - m_new) : 1.0f;
      if (need) {
        l *= alpha;
        m_ref = m_new;
      }
      // P = 2^(S * scale * log2e - m_ref), row sum, bf16 P back over S (32 keys -> 16 columns at a time)
      // a row that has seen no key yet (m_ref = -inf; causal with N > Nk) has only masked scores
      const float m_sub = GEN && m_ref == -INFINITY ? 0.0f : m_ref;
      const float2 c2 = make_float2(sl2, sl2), nm2 = make_float2(-m_sub, -m_sub);
      float2 ls0 = make_float2(0.f, 0.f), ls1 = make_float2(0.f, 0.f);
      // POLY16 of every 16 element pairs (evenly spaced) take the cubic
      constexpr int kPolyStride = POLY16 > 0 ? 16 / POLY16 : 16;
      // The two paths are separate code, so the tiles that use the cubic for part of their
      // exponentials issue no SFU operation for that part (a select between the two would).
      auto exp_store = [&](auto poly_tag) {
        constexpr bool kPoly = decltype(poly_tag)::value;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int c = 32 * cc + 2 * e;
            const float2 x = __ffma2_rn(make_float2(S(c), S(c + 1)), c2, nm2);
            float2 p;
            if (kPoly && e % kPolyStride == 0) {
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
          tmem_st16(tS + 16 * cc, pk);
        }
      };
      if (POLY16 > 0 && !edge)  // masked (edge) tiles keep exact zeros from the SFU
        exp_store(std::true_type{});
      else
        exp_store(std::false_type{});
#undef S
      const float2 ls = __fadd2_rn(ls0, ls1);
      l += ls.x + ls.y;
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        // correction: this thread's row of O_t *= alpha once the previous P.V has landed (before
        // p_full lets the next P.V accumulate into it)
        ok = wait_warp(&o_full[t], (j - 1) & 1, g, kSiteFwd | 8);
        tc_fence_after();
        if (ok) {
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tO + 32 * c, o);
            tmem_wait_ld();
            reg_fence(o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + 32 * c, o);
          }
        }
      }
      tmem_wait_st();
      tc_fence_before();
      if (!ok) break;
      mbar_arrive(&p_full[t]);
    }
    if (ok && nkv[t] > 0) ok = wait_warp(&o_full[t], (nkv[t] - 1) & 1, g, kSiteFwd | 9);
    if (ok && nkv[t] > 0 && prm.O_acc != nullptr) {
      // fold into the fp32 accumulators: L = ln(e^LSE_old + e^LSE), O_acc = e^(LSE_old - L) O_acc +
      // e^(LSE - L) O (a side at -inf weighs 0; both at -inf leave O_acc = 0, LSE_acc = -inf); the
      // row's thread alone reads and replaces its LSE
      tc_fence_after();
      const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;
      const bool store = row < prm.N;
      const size_t ri = static_cast<size_t>(bh) * prm.N + (store ? row : 0);
      const float lse = l > 0.0f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
      float lse_new = lse, wa = 0.0f, wb = 1.0f;
      if (!prm.acc_first && store) {
        const float lse_old = prm.LSE_acc[ri];
        const float mx = fmaxf(lse_old, lse);
        lse_new = mx == -INFINITY ? -INFINITY : mx + log1pf(expf(-fabsf(lse_old - lse)));
        wa = lse_new == -INFINITY ? 0.0f : expf(lse_old - lse_new);
        wb = lse_new == -INFINITY ? 0.0f : expf(lse - lse_new);
      }
      const float scale_b = inv_l * wb;
      float* arow = prm.O_acc + ri * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t o[32];
        tmem_ld32(tO + 32 * c, o);
        tmem_wait_ld();
        reg_fence(o);
        if (store) {
          float4* dst = reinterpret_cast<float4*>(arow + 32 * c);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            float4 v = make_float4(__uint_as_float(o[4 * i]) * scale_b, __uint_as_float(o[4 * i + 1]) * scale_b,
                                   __uint_as_float(o[4 * i + 2]) * scale_b, __uint_as_float(o[4 * i + 3]) * scale_b);
            if (!prm.acc_first) {
              const float4 a = dst[i];
              v.x = fmaf(wa, a.x, v.x);
              v.y = fmaf(wa, a.y, v.y);
              v.z = fmaf(wa, a.z, v.z);
              v.w = fmaf(wa, a.w, v.w);
            }
            dst[i] = v;
          }
        }
      }
      if (store) prm.LSE_acc[ri] = lse_new;
    } else if (ok && nkv[t] > 0) {
      tc_fence_after();
      const float inv_l = l > 0.0f ? 1.0f / l : 0.0f;  // a row that sees no key: O = 0, LSE = -inf
      const bool store = row < prm.N;
      __nv_bfloat16* orow = prm.O + (static_cast<size_t>(bh) * prm.N + (store ? row : 0)) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
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
      if (store)
        prm.LSE[static_cast<size_t>(bh) * prm.N + row] =
            l > 0.0f ? (m_ref + log2f(l)) * 0.69314718055994531f : -INFINITY;
    } else if (nkv[t] == 0 && qt < n_tiles && row < prm.N) {
      // a query tile no key is visible to (causal, N > Nk): O = 0, LSE = -inf (an accumulating call
      // that is not the first adds nothing)
      if (prm.O_acc == nullptr) {
        __nv_bfloat16* orow = prm.O + (static_cast<size_t>(bh) * prm.N + row) * D;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) reinterpret_cast<uint4*>(orow)[i] = make_uint4(0u, 0u, 0u, 0u);
        prm.LSE[static_cast<size_t>(bh) * prm.N + row] = -INFINITY;
      } else if (prm.acc_first) {
        float* arow = prm.O_acc + (static_cast<size_t>(bh) * prm.N + row) * D;
#pragma unroll
        for (int i = 0; i < D / 4; ++i) reinterpret_cast<float4*>(arow)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        prm.LSE_acc[static_cast<size_t>(bh) * prm.N + row] = -INFINITY;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace fa
