// fa_api.cu -- host side of libfa: argument checks, TMA descriptors, launches.
// See include/fa.h for the contract of every entry point.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/fa.h"
#include "exp2_poly.cuh"
#include "fa_bwd.cuh"
#include "fa_bwd2.cuh"
#include "fa_fwd.cuh"
#include "fa_fwd2.cuh"
#include "fa_merge.cuh"

namespace {

constexpr int kMaxDevices = 64;
// Forward: element pairs out of every 16 whose exponentials take the FMA-pipe cubic by default,
// per head dimension (index 0: d = 64, 1: d = 128).
constexpr int kPolyDefault[2] = {4, 1};
constexpr int kBwdPoly16 = 0;  // backward: the SFU alone measured faster than any polynomial share

__device__ int g_status;  // first device-side failure (wait site), 0 = none

struct DeviceState {
  std::once_flag once;
  int* status = nullptr;
  cudaError_t err = cudaSuccess;
};
DeviceState g_dev[kMaxDevices];

// Process-wide switches (atomics: a setter racing with calls on other threads is not a data race;
// which setting a concurrent call sees is unspecified).
std::atomic<float> g_tau{fa::kRescaleTau};
std::atomic<int> g_poly{-1};      // cubic pairs per 16 in the forward; -1 = kPolyDefault for the head dimension
std::atomic<int> g_fwd_pair{0};   // 1: forward at d = 128 on cluster pairs (cta_group::2 UMMA)
std::atomic<int> g_bwd_pair{0};   // 1: backward at d = 128 on cluster pairs (cta_group::2 UMMA)
// One-shot profiling events [fwd|bwd][start|stop], per host thread: armed by fa_profile_next and
// consumed by the next fa_fwd* / fa_bwd* call made on the same thread.
thread_local cudaEvent_t g_prof[2][2] = {{nullptr, nullptr}, {nullptr, nullptr}};

// Records the pending start event of `which` (if any) on `st`; returns whether one was pending.
bool prof_begin(int which, cudaStream_t st) {
  if (!g_prof[which][0]) return false;
  cudaEventRecord(g_prof[which][0], st);
  return true;
}
void prof_end(int which, cudaStream_t st) {
  if (g_prof[which][1]) cudaEventRecord(g_prof[which][1], st);
  g_prof[which][0] = g_prof[which][1] = nullptr;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Status word of the current device (set up once per device).
int* device_status(int* err_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err_out = FA_ERR_CUDA;
    return nullptr;
  }
  DeviceState& s = g_dev[dev];
  std::call_once(s.once, [&s] {
    void* p = nullptr;
    s.err = cudaGetSymbolAddress(&p, g_status);
    if (s.err == cudaSuccess) s.status = static_cast<int*>(p);
  });
  if (!s.status) *err_out = FA_ERR_CUDA;
  return s.status;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

// Encoded tensor maps of recent calls, keyed by (address, extents, box, element kind): callers that
// reuse their buffers (training loops, graph replays, the ring steps) skip cuTensorMapEncodeTiled.
// A map holds only the address and geometry it was encoded from, so a hit is exactly the map a
// fresh encode would produce.  Small, round-robin replacement, one lock.
struct MapKey {
  const void* base;
  int BH, N, d, rows, kind;  // kind 0: bf16 operand, 1: fp32 dQ accumulator
  bool operator==(const MapKey& o) const {
    return base == o.base && BH == o.BH && N == o.N && d == o.d && rows == o.rows && kind == o.kind;
  }
};
struct MapCache {
  static constexpr int kSlots = 64;
  std::mutex mu;
  MapKey key[kSlots] = {};
  CUtensorMap map[kSlots];
  int used = 0, next = 0;
};
MapCache g_maps;

bool map_lookup(const MapKey& k, CUtensorMap* out) {
  std::lock_guard<std::mutex> lock(g_maps.mu);
  for (int i = 0; i < g_maps.used; ++i)
    if (g_maps.key[i] == k) {
      *out = g_maps.map[i];
      return true;
    }
  return false;
}
void map_store(const MapKey& k, const CUtensorMap& m) {
  std::lock_guard<std::mutex> lock(g_maps.mu);
  const int i = g_maps.used < MapCache::kSlots ? g_maps.used++ : g_maps.next;
  if (i == g_maps.next) g_maps.next = (g_maps.next + 1) % MapCache::kSlots;
  g_maps.key[i] = k;
  g_maps.map[i] = m;
}

// 3-D map over a contiguous [BH, N, d] bf16 tensor: box 64 (d) x `rows` x 1, 128-byte swizzle.
bool make_map(CUtensorMap* map, const void* base, int BH, int N, int d, int rows = 128) {
  const MapKey key{base, BH, N, d, rows, 0};
  if (map_lookup(key, map)) return true;
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(N) * d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  map_store(key, *map);
  return true;
}

// 3-D map over the fp32 dQ accumulator [BH, Npad, d]: box 32 (d) x `rows` x 1, 128-byte swizzle
// (the layout of the backward kernels' staging buffers for their TMA reduce-add).
bool make_acc_map(CUtensorMap* map, void* base, int BH, int npad, int d, int rows = 128) {
  const MapKey key{base, BH, npad, d, rows, 1};
  if (map_lookup(key, map)) return true;
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(npad),
                              static_cast<cuuint64_t>(BH)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 4, static_cast<cuuint64_t>(npad) * d * 4};
  const cuuint32_t box[3] = {32, static_cast<cuuint32_t>(rows), 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  if (fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  map_store(key, *map);
  return true;
}

// Shape checks shared by forward and backward (Hq query heads over Hkv key/value heads, Nq query
// and Nk key rows).  Returns FA_OK, or the error; *empty set for 0-size problems.
int check_shape(int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, bool* empty) {
  *empty = false;
  if (B < 0 || Hq < 0 || Hkv < 0 || Nq < 0 || Nk < 0) return FA_ERR_INVALID_ARG;
  if (causal != 0 && causal != 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.0f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (Hkv == 0 ? Hq != 0 : Hq % Hkv != 0) return FA_ERR_INVALID_ARG;
  if (B == 0 || Hq == 0 || Nq == 0) {
    *empty = true;
    return FA_OK;
  }
  if (Nk == 0) return FA_ERR_INVALID_ARG;  // every query needs a key set to attend to
  for (const long long N : {static_cast<long long>(Nq), static_cast<long long>(Nk)}) {
    const long long BH = static_cast<long long>(B) * (N == Nq ? Hq : Hkv);
    const long long tiles = (N + 127) / 128;
    // grid size, tensor-map extents and int row indices must stay in range
    if (BH > INT_MAX / 2 || BH * tiles > INT_MAX || N + 128 > INT_MAX) return FA_ERR_UNSUPPORTED;
    if (BH * (tiles * 128) * d > (1LL << 46)) return FA_ERR_UNSUPPORTED;
  }
  if (static_cast<long long>(B) * Hq * ((Nq + 127) / 128) > INT_MAX) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

// The dynamic shared memory limit of a kernel is a per-device attribute: set it once per (kernel,
// device) and remember that it is set.
std::mutex g_attr_mu;
struct AttrDone {
  const void* kernel;
  int device;
};
AttrDone g_attr_done[256];
int g_attr_count = 0;

template <typename K>
cudaError_t set_smem(K kernel, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const void* key = reinterpret_cast<const void*>(kernel);
  std::lock_guard<std::mutex> lock(g_attr_mu);
  for (int i = 0; i < g_attr_count; ++i)
    if (g_attr_done[i].kernel == key && g_attr_done[i].device == dev) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && g_attr_count < 256) g_attr_done[g_attr_count++] = AttrDone{key, dev};
  return e;
}

template <int D, bool C, int P>
int launch_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const fa::FwdParams& prm,
               cudaStream_t st) {
  using L = fa::FwdLayout<D>;
  const bool gen = prm.G != 1 || prm.Nk != prm.N;
  auto kern = gen ? fa::fwd_kernel<D, C, P, true> : fa::fwd_kernel<D, C, P, false>;
  if (set_smem(kern, L::kBytes) != cudaSuccess) return FA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(prm.BH) * static_cast<unsigned>(prm.n_pairs);
  kern<<<grid, L::kThreads, L::kBytes, st>>>(q, k, v, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool C, int P>
int launch_fwd2(const CUtensorMap& q, const CUtensorMap& k64, const CUtensorMap& v, const fa::Fwd2Params& prm,
                cudaStream_t st) {
  auto kern = fa::fwd2_kernel<C, P>;
  if (set_smem(kern, fa::Fwd2Layout::kBytes) != cudaSuccess) return FA_ERR_CUDA;
  const unsigned grid = 2u * static_cast<unsigned>(prm.BH) * static_cast<unsigned>(prm.n_quads);
  kern<<<grid, fa::Fwd2Layout::kThreads, fa::Fwd2Layout::kBytes, st>>>(q, k64, v, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// The forward with `poly` (0, 1, 2 or 4) of every 16 element pairs on the cubic.
template <int D, bool C>
int launch_fwd_poly(int poly, const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                    const fa::FwdParams& prm, cudaStream_t st) {
  switch (poly) {
    case 0: return launch_fwd<D, C, 0>(q, k, v, prm, st);
    case 1: return launch_fwd<D, C, 1>(q, k, v, prm, st);
    case 2: return launch_fwd<D, C, 2>(q, k, v, prm, st);
    default: return launch_fwd<D, C, 4>(q, k, v, prm, st);
  }
}

template <bool C>
int launch_fwd2_poly(int poly, const CUtensorMap& q, const CUtensorMap& k64, const CUtensorMap& v,
                     const fa::Fwd2Params& prm, cudaStream_t st) {
  switch (poly) {
    case 0: return launch_fwd2<C, 0>(q, k64, v, prm, st);
    case 1: return launch_fwd2<C, 1>(q, k64, v, prm, st);
    case 2: return launch_fwd2<C, 2>(q, k64, v, prm, st);
    default: return launch_fwd2<C, 4>(q, k64, v, prm, st);
  }
}

template <int D, bool C>
int launch_bwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v, const CUtensorMap& dO,
               const CUtensorMap& dq_acc, const fa::BwdParams& prm, cudaStream_t st) {
  using L = fa::BwdLayout<D>;
  const bool gen = prm.G != 1 || prm.Nk != prm.N;
  auto kern = gen ? fa::bwd_kernel<D, C, kBwdPoly16, true> : fa::bwd_kernel<D, C, kBwdPoly16, false>;
  if (set_smem(kern, L::kBytes) != cudaSuccess) return FA_ERR_CUDA;
  const unsigned grid = static_cast<unsigned>(prm.BHkv) * static_cast<unsigned>(prm.n_kv_tiles);
  kern<<<grid, L::kThreads, L::kBytes, st>>>(q, k, v, dO, dq_acc, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

template <bool C>
int launch_bwd2(const CUtensorMap& q, const CUtensorMap& q64, const CUtensorMap& k, const CUtensorMap& v,
                const CUtensorMap& dO, const CUtensorMap& dO64, const CUtensorMap& dq_acc64, const fa::BwdParams& prm,
                cudaStream_t st) {
  auto kern = fa::bwd2_kernel<C>;
  if (set_smem(kern, fa::Bwd2Layout::kBytes) != cudaSuccess) return FA_ERR_CUDA;
  const unsigned grid = 2u * static_cast<unsigned>(prm.BHkv) * static_cast<unsigned>((prm.n_kv_tiles + 1) / 2);
  kern<<<grid, 384, fa::Bwd2Layout::kBytes, st>>>(q, q64, k, v, dO, dO64, dq_acc64, prm);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

struct WsLayout {
  size_t dq, lse2, dsum, total;
};
size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
WsLayout ws_layout(long long BH, int N, int d) {
  const size_t npad = static_cast<size_t>((N + 127) / 128) * 128;
  WsLayout w;
  w.dq = 0;
  w.lse2 = round256(static_cast<size_t>(BH) * npad * d * sizeof(float));
  w.dsum = w.lse2 + round256(static_cast<size_t>(BH) * npad * sizeof(float));
  w.total = w.dsum + round256(static_cast<size_t>(BH) * npad * sizeof(float));
  return w;
}

// One CTA waits on a barrier that never completes: exercises the bounded-wait failure path.
__global__ void selftest_wait_kernel(int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    fa::mbar_init(&bar, 1);
    abort_flag = 0;
    fa::fence_mbar_init();
  }
  __syncthreads();
  const fa::Guard g{&abort_flag, status};
  fa::wait_warp(&bar, 0, g, 0xF01);  // nobody arrives: gives up after the wait limit
  __syncthreads();
  if (threadIdx.x == 0) fa::mbar_arrive(&bar);  // complete the phase so the barrier is left idle
}

// One thread: SM cycles elapsed while the global timer advances by 20 us (a bounded spin).
__global__ void clock_probe_kernel(unsigned long long* out) {
  const unsigned long long t0 = fa::globaltimer();
  const long long c0 = clock64();
  unsigned long long t1 = t0;
  while (t1 - t0 < 20000ull) t1 = fa::globaltimer();
  const long long c1 = clock64();
  out[0] = static_cast<unsigned long long>(c1 - c0);
  out[1] = t1 - t0;
}

__global__ void exp2_eval_kernel(const float* __restrict__ x, float* __restrict__ y, long long n, int mode) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n) return;
  if (mode == 2) {  // packed form: lane i&1 of the pair (i & ~1, i | 1)
    const long long i1 = (i | 1) < n ? (i | 1) : i;
    const float2 r = fa::exp2_poly2(make_float2(x[i & ~1LL], x[i1]));
    y[i] = (i & 1) ? r.y : r.x;
  } else {
    y[i] = mode == 0 ? fa::exp2_poly(x[i]) : fa::exp2_sfu(x[i]);
  }
}

// True when any of the `no` output ranges overlaps an input range or another output range.
bool any_overlap(const void* const* outs, const size_t* osz, int no, const void* const* ins, const size_t* isz, int ni) {
  for (int a = 0; a < no; ++a) {
    for (int b = 0; b < ni; ++b)
      if (overlaps(outs[a], osz[a], ins[b], isz[b])) return true;
    for (int b = a + 1; b < no; ++b)
      if (overlaps(outs[a], osz[a], outs[b], osz[b])) return true;
  }
  return false;
}

// The forward after its argument checks: bf16 O and LSE, or (O_acc non-null) the fold into fp32
// accumulators.  The cluster-pair variant serves only plain bf16 calls.
int fwd_launch(const void* Q, const void* K, const void* V, void* O, float* LSE, float* O_acc, float* LSE_acc,
               int acc_first, int B, int Hq, int Hkv, int Nq, int Nk, int d, float scale, int causal, void* stream) {
  int rc = FA_OK;
  int* status = device_status(&rc);
  if (!status) return rc;
  const int BH = B * Hq, BHkv = B * Hkv;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, BH, Nq, d) || !make_map(&mk, K, BHkv, Nk, d) || !make_map(&mv, V, BHkv, Nk, d))
    return FA_ERR_CUDA;
  fa::FwdParams prm;
  prm.O = static_cast<__nv_bfloat16*>(O);
  prm.LSE = LSE;
  prm.O_acc = O_acc;
  prm.LSE_acc = LSE_acc;
  prm.acc_first = acc_first;
  prm.N = Nq;
  prm.Nk = Nk;
  prm.BH = BH;
  prm.Hq = Hq;
  prm.G = Hq / Hkv;
  prm.off = Nk - Nq;
  const int tiles = (Nq + 127) / 128;
  prm.n_pairs = (tiles + 1) / 2;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.tau = g_tau.load(std::memory_order_relaxed);
  prm.status = status;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int poly_set = g_poly.load(std::memory_order_relaxed);
  const int poly = poly_set >= 0 ? poly_set : kPolyDefault[d == 128 ? 1 : 0];
  if (!O_acc && d == 128 && g_fwd_pair.load(std::memory_order_relaxed) && Hq == Hkv && Nq == Nk) {
    CUtensorMap mk64;
    if (!make_map(&mk64, K, BH, Nk, d, 64)) return FA_ERR_CUDA;
    fa::Fwd2Params p2;
    p2.O = prm.O;
    p2.LSE = prm.LSE;
    p2.N = Nq;
    p2.BH = BH;
    p2.n_quads = (tiles + 3) / 4;
    p2.scale_log2 = prm.scale_log2;
    p2.tau = prm.tau;
    p2.status = prm.status;
    const bool prof2 = prof_begin(0, st);
    rc = causal ? launch_fwd2_poly<true>(poly, mq, mk64, mv, p2, st) : launch_fwd2_poly<false>(poly, mq, mk64, mv, p2, st);
    if (prof2) prof_end(0, st);
    return rc;
  }
  const bool prof = prof_begin(0, st);
  if (d == 128)
    rc = causal ? launch_fwd_poly<128, true>(poly, mq, mk, mv, prm, st)
                : launch_fwd_poly<128, false>(poly, mq, mk, mv, prm, st);
  else
    rc = causal ? launch_fwd_poly<64, true>(poly, mq, mk, mv, prm, st)
                : launch_fwd_poly<64, false>(poly, mq, mk, mv, prm, st);
  if (prof) prof_end(0, st);
  return rc;
}

// Backward step 1: -D_i, -LSE_i * log2(e) for every (padded) query row and the fp32 dQ accumulator
// zeroed, all in the workspace.
int bwd_prep_launch(const void* O, const void* dO, const float* LSE, uint8_t* wsb, const WsLayout& ws, int BH, int Nq,
                    int d, cudaStream_t st) {
  const int npad = (Nq + 127) / 128 * 128;
  const long long prep_rows = static_cast<long long>(BH) * npad;
  const unsigned prep_grid = static_cast<unsigned>((prep_rows * (d / 8) + 255) / 256);
  float* dq_acc = reinterpret_cast<float*>(wsb + ws.dq);
  float* lse2 = reinterpret_cast<float*>(wsb + ws.lse2);
  float* dsum = reinterpret_cast<float*>(wsb + ws.dsum);
  const auto* o = static_cast<const __nv_bfloat16*>(O);
  const auto* g = static_cast<const __nv_bfloat16*>(dO);
  if (d == 128)
    fa::bwd_prep_kernel<128><<<prep_grid, 256, 0, st>>>(o, g, LSE, lse2, dsum, dq_acc, Nq, npad, prep_rows);
  else
    fa::bwd_prep_kernel<64><<<prep_grid, 256, 0, st>>>(o, g, LSE, lse2, dsum, dq_acc, Nq, npad, prep_rows);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

// Backward step 2: the main kernel over one key block.  dQ adds into the workspace accumulator;
// dK and dV are written as bf16 (dK, dV) or added to fp32 accumulators (dK_acc, dV_acc).
int bwd_main_launch(const void* Q, const void* K, const void* V, const void* dO, uint8_t* wsb, const WsLayout& ws,
                    void* dK, void* dV, float* dK_acc, float* dV_acc, int acc_first, int B, int Hq, int Hkv, int Nq,
                    int Nk, int d, float scale, int causal, int* status, cudaStream_t st, bool allow_pair) {
  const int BH = B * Hq, BHkv = B * Hkv;
  const int q_tiles = (Nq + 127) / 128;
  const int npad = q_tiles * 128;
  float* dq_acc = reinterpret_cast<float*>(wsb + ws.dq);
  CUtensorMap mq, mk, mv, mdo, macc;
  if (!make_map(&mq, Q, BH, Nq, d) || !make_map(&mk, K, BHkv, Nk, d) || !make_map(&mv, V, BHkv, Nk, d) ||
      !make_map(&mdo, dO, BH, Nq, d) || !make_acc_map(&macc, dq_acc, BH, npad, d))
    return FA_ERR_CUDA;
  fa::BwdParams prm;
  prm.nlse2 = reinterpret_cast<const float*>(wsb + ws.lse2);
  prm.ndsum = reinterpret_cast<const float*>(wsb + ws.dsum);
  prm.dK = static_cast<__nv_bfloat16*>(dK);
  prm.dV = static_cast<__nv_bfloat16*>(dV);
  prm.dK_acc = dK_acc;
  prm.dV_acc = dV_acc;
  prm.acc_first = acc_first;
  prm.N = Nq;
  prm.Npad = npad;
  prm.Nk = Nk;
  prm.BHkv = BHkv;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.G = Hq / Hkv;
  prm.off = Nk - Nq;
  prm.n_q_tiles = q_tiles;
  prm.n_kv_tiles = (Nk + 127) / 128;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.scale = scale;
  prm.status = status;
  int rc = FA_OK;
  const bool prof = prof_begin(1, st);
  if (allow_pair && d == 128 && g_bwd_pair.load(std::memory_order_relaxed) && Hq == Hkv && Nq == Nk) {
    CUtensorMap mq64, mdo64, macc64;
    if (!make_map(&mq64, Q, BH, Nq, d, 64) || !make_map(&mdo64, dO, BH, Nq, d, 64) ||
        !make_acc_map(&macc64, dq_acc, BH, npad, d, 64))
      rc = FA_ERR_CUDA;
    else
      rc = causal ? launch_bwd2<true>(mq, mq64, mk, mv, mdo, mdo64, macc64, prm, st)
                  : launch_bwd2<false>(mq, mq64, mk, mv, mdo, mdo64, macc64, prm, st);
  } else if (d == 128) {
    rc = causal ? launch_bwd<128, true>(mq, mk, mv, mdo, macc, prm, st)
                : launch_bwd<128, false>(mq, mk, mv, mdo, macc, prm, st);
  } else {
    rc = causal ? launch_bwd<64, true>(mq, mk, mv, mdo, macc, prm, st)
                : launch_bwd<64, false>(mq, mk, mv, mdo, macc, prm, st);
  }
  if (prof) prof_end(1, st);
  return rc;
}

// Backward step 3: dQ = bf16(scale * dQ_acc) for the real rows.
int bwd_finish_launch(uint8_t* wsb, const WsLayout& ws, void* dQ, int BH, int Nq, int d, float scale, cudaStream_t st) {
  const int npad = (Nq + 127) / 128 * 128;
  const float* dq_acc = reinterpret_cast<const float*>(wsb + ws.dq);
  const long long rows = static_cast<long long>(BH) * Nq;
  const unsigned cgrid = static_cast<unsigned>((rows * (d / 8) + 255) / 256);
  if (d == 128)
    fa::bwd_dq_kernel<128><<<cgrid, 256, 0, st>>>(dq_acc, static_cast<__nv_bfloat16*>(dQ), scale, Nq, npad, rows);
  else
    fa::bwd_dq_kernel<64><<<cgrid, 256, 0, st>>>(dq_acc, static_cast<__nv_bfloat16*>(dQ), scale, Nq, npad, rows);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace

extern "C" {

int fa_version(void) { return 100; }

const char* fa_strerror(int status) {
  switch (status) {
    case FA_OK: return "ok";
    case FA_ERR_INVALID_ARG: return "invalid argument";
    case FA_ERR_UNSUPPORTED: return "unsupported shape or head dimension";
    case FA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case FA_ERR_CUDA: return "CUDA error";
    case FA_ERR_TIMEOUT: return "device pipeline wait timed out";
    default: return "unknown status";
  }
}

int fa_set_softmax_options(float tau, int poly) {
  if (!(tau >= 0.0f && tau <= 16.0f) || (poly != -1 && poly != 0 && poly != 1 && poly != 2 && poly != 4))
    return FA_ERR_INVALID_ARG;
  g_tau = tau;
  g_poly = poly;
  return FA_OK;
}

int fa_fwd_qk(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int Hq, int Hkv, int Nq,
              int Nk, int d, float scale, int causal, void* stream) {
  bool empty = false;
  int rc = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal, &empty);
  if (rc != FA_OK) return rc;
  if (!Q || !K || !V || !O || !LSE) return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(LSE)) return FA_ERR_ALIGNMENT;
  const int BH = B * Hq, BHkv = B * Hkv;
  const size_t qb = static_cast<size_t>(BH) * Nq * d * 2, kb = static_cast<size_t>(BHkv) * Nk * d * 2;
  const size_t lb = static_cast<size_t>(BH) * Nq * 4;
  const void* outs[2] = {O, LSE};
  const size_t osz[2] = {qb, lb};
  const void* ins[3] = {Q, K, V};
  const size_t isz[3] = {qb, kb, kb};
  if (any_overlap(outs, osz, 2, ins, isz, 3)) return FA_ERR_INVALID_ARG;
  return fwd_launch(Q, K, V, O, LSE, nullptr, nullptr, 0, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream);
}

int fa_fwd_accumulate(const void* Q, const void* K, const void* V, float* O_acc, float* LSE_acc, int B, int Hq,
                      int Hkv, int Nq, int Nk, int d, float scale, int causal, int first, void* stream) {
  bool empty = false;
  int rc = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal, &empty);
  if (rc != FA_OK) return rc;
  if (first != 0 && first != 1) return FA_ERR_INVALID_ARG;
  if (!Q || !K || !V || !O_acc || !LSE_acc) return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O_acc) || !aligned16(LSE_acc))
    return FA_ERR_ALIGNMENT;
  const int BH = B * Hq, BHkv = B * Hkv;
  const size_t qb = static_cast<size_t>(BH) * Nq * d * 2, kb = static_cast<size_t>(BHkv) * Nk * d * 2;
  const size_t lb = static_cast<size_t>(BH) * Nq * 4;
  const void* outs[2] = {O_acc, LSE_acc};
  const size_t osz[2] = {2 * qb, lb};
  const void* ins[3] = {Q, K, V};
  const size_t isz[3] = {qb, kb, kb};
  if (any_overlap(outs, osz, 2, ins, isz, 3)) return FA_ERR_INVALID_ARG;
  return fwd_launch(Q, K, V, nullptr, nullptr, O_acc, LSE_acc, first, B, Hq, Hkv, Nq, Nk, d, scale, causal, stream);
}

int fa_fwd(const void* Q, const void* K, const void* V, void* O, float* LSE, int B, int H, int N, int d,
           float scale, int causal, void* stream) {
  return fa_fwd_qk(Q, K, V, O, LSE, B, H, H, N, N, d, scale, causal, stream);
}

size_t fa_bwd_qk_workspace_size(int B, int Hq, int Nq, int d) {
  bool empty = false;
  if (check_shape(B, Hq, Hq, Nq, Nq, d, 1.0f, 0, &empty) != FA_OK || empty) return 0;
  return ws_layout(static_cast<long long>(B) * Hq, Nq, d).total;
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) { return fa_bwd_qk_workspace_size(B, H, N, d); }

int fa_bwd_qk(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE, void* dQ,
              void* dK, void* dV, void* workspace, size_t workspace_bytes, int B, int Hq, int Hkv, int Nq, int Nk,
              int d, float scale, int causal, void* stream) {
  bool empty = false;
  int rc = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal, &empty);
  if (rc != FA_OK) return rc;
  if (!Q || !K || !V || !O || !dO || !LSE || !dQ || !dK || !dV || !workspace) return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  for (const void* p : {Q, K, V, O, dO, static_cast<const void*>(LSE), static_cast<const void*>(dQ),
                        static_cast<const void*>(dK), static_cast<const void*>(dV), static_cast<const void*>(workspace)})
    if (!aligned16(p)) return FA_ERR_ALIGNMENT;
  const int BH = B * Hq, BHkv = B * Hkv;
  const WsLayout ws = ws_layout(BH, Nq, d);
  if (workspace_bytes < ws.total) return FA_ERR_INVALID_ARG;
  const size_t qb = static_cast<size_t>(BH) * Nq * d * 2, kb = static_cast<size_t>(BHkv) * Nk * d * 2;
  const size_t lb = static_cast<size_t>(BH) * Nq * 4;
  const void* outs[4] = {dQ, dK, dV, workspace};
  const size_t osz[4] = {qb, kb, kb, ws.total};
  const void* ins[6] = {Q, K, V, O, dO, LSE};
  const size_t isz[6] = {qb, kb, kb, qb, qb, lb};
  if (any_overlap(outs, osz, 4, ins, isz, 6)) return FA_ERR_INVALID_ARG;
  int* status = device_status(&rc);
  if (!status) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  if ((rc = bwd_prep_launch(O, dO, LSE, wsb, ws, BH, Nq, d, st)) != FA_OK) return rc;
  if ((rc = bwd_main_launch(Q, K, V, dO, wsb, ws, dK, dV, nullptr, nullptr, 0, B, Hq, Hkv, Nq, Nk, d, scale, causal,
                            status, st, true)) != FA_OK)
    return rc;
  return bwd_finish_launch(wsb, ws, dQ, BH, Nq, d, scale, st);
}

int fa_bwd_prepare(const void* O, const void* dO, const float* LSE, void* workspace, size_t workspace_bytes, int B,
                   int Hq, int Nq, int d, void* stream) {
  bool empty = false;
  int rc = check_shape(B, Hq, Hq, Nq, Nq, d, 1.0f, 0, &empty);
  if (rc != FA_OK) return rc;
  if (!O || !dO || !LSE || !workspace) return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  for (const void* p : {O, dO, static_cast<const void*>(LSE), static_cast<const void*>(workspace)})
    if (!aligned16(p)) return FA_ERR_ALIGNMENT;
  const int BH = B * Hq;
  const WsLayout ws = ws_layout(BH, Nq, d);
  if (workspace_bytes < ws.total) return FA_ERR_INVALID_ARG;
  const size_t qb = static_cast<size_t>(BH) * Nq * d * 2, lb = static_cast<size_t>(BH) * Nq * 4;
  const void* outs[1] = {workspace};
  const size_t osz[1] = {ws.total};
  const void* ins[3] = {O, dO, LSE};
  const size_t isz[3] = {qb, qb, lb};
  if (any_overlap(outs, osz, 1, ins, isz, 3)) return FA_ERR_INVALID_ARG;
  return bwd_prep_launch(O, dO, LSE, static_cast<uint8_t*>(workspace), ws, BH, Nq, d,
                         static_cast<cudaStream_t>(stream));
}

int fa_bwd_accumulate(const void* Q, const void* K, const void* V, const void* dO, void* workspace,
                      size_t workspace_bytes, float* dK_acc, float* dV_acc, int B, int Hq, int Hkv, int Nq, int Nk,
                      int d, float scale, int causal, int first, void* stream) {
  bool empty = false;
  int rc = check_shape(B, Hq, Hkv, Nq, Nk, d, scale, causal, &empty);
  if (rc != FA_OK) return rc;
  if (first != 0 && first != 1) return FA_ERR_INVALID_ARG;
  if (!Q || !K || !V || !dO || !workspace || !dK_acc || !dV_acc) return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  for (const void* p : {Q, K, V, dO, static_cast<const void*>(workspace), static_cast<const void*>(dK_acc),
                        static_cast<const void*>(dV_acc)})
    if (!aligned16(p)) return FA_ERR_ALIGNMENT;
  const int BH = B * Hq, BHkv = B * Hkv;
  const WsLayout ws = ws_layout(BH, Nq, d);
  if (workspace_bytes < ws.total) return FA_ERR_INVALID_ARG;
  const size_t qb = static_cast<size_t>(BH) * Nq * d * 2, kb = static_cast<size_t>(BHkv) * Nk * d * 2;
  const void* outs[3] = {workspace, dK_acc, dV_acc};
  const size_t osz[3] = {ws.total, 2 * kb, 2 * kb};
  const void* ins[4] = {Q, K, V, dO};
  const size_t isz[4] = {qb, kb, kb, qb};
  if (any_overlap(outs, osz, 3, ins, isz, 4)) return FA_ERR_INVALID_ARG;
  int* status = device_status(&rc);
  if (!status) return rc;
  return bwd_main_launch(Q, K, V, dO, static_cast<uint8_t*>(workspace), ws, nullptr, nullptr, dK_acc, dV_acc, first, B,
                         Hq, Hkv, Nq, Nk, d, scale, causal, status, static_cast<cudaStream_t>(stream), false);
}

int fa_bwd_finish(void* workspace, size_t workspace_bytes, void* dQ, int B, int Hq, int Nq, int d, float scale,
                  void* stream) {
  bool empty = false;
  int rc = check_shape(B, Hq, Hq, Nq, Nq, d, scale, 0, &empty);
  if (rc != FA_OK) return rc;
  if (!workspace || !dQ) return FA_ERR_INVALID_ARG;
  if (empty) return FA_OK;
  if (!aligned16(workspace) || !aligned16(dQ)) return FA_ERR_ALIGNMENT;
  const int BH = B * Hq;
  const WsLayout ws = ws_layout(BH, Nq, d);
  if (workspace_bytes < ws.total) return FA_ERR_INVALID_ARG;
  if (overlaps(dQ, static_cast<size_t>(BH) * Nq * d * 2, workspace, ws.total)) return FA_ERR_INVALID_ARG;
  return bwd_finish_launch(static_cast<uint8_t*>(workspace), ws, dQ, BH, Nq, d, scale,
                           static_cast<cudaStream_t>(stream));
}

int fa_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE, void* dQ,
           void* dK, void* dV, void* workspace, size_t workspace_bytes, int B, int H, int N, int d, float scale,
           int causal, void* stream) {
  return fa_bwd_qk(Q, K, V, O, dO, LSE, dQ, dK, dV, workspace, workspace_bytes, B, H, H, N, N, d, scale, causal,
                   stream);
}

}  // extern "C"

namespace {

// Scratch for fa_bwd_noalloc: a fixed device array instead of a caller workspace.
__device__ __align__(256) unsigned char g_noalloc_scratch[FA_BWD_NOALLOC_SCRATCH_BYTES];

struct ScratchState {
  std::once_flag once;
  void* ptr = nullptr;
};
ScratchState g_scratch[kMaxDevices];

// Device address of g_noalloc_scratch on the current device (looked up once per device;
// in host code the symbol itself is only a host-side stand-in, never a device address).
void* noalloc_scratch(int* err_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *err_out = FA_ERR_CUDA;
    return nullptr;
  }
  ScratchState& s = g_scratch[dev];
  std::call_once(s.once, [&s] {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) == cudaSuccess) s.ptr = p;
  });
  if (!s.ptr) *err_out = FA_ERR_CUDA;
  return s.ptr;
}

}  // namespace

extern "C" {

int fa_bwd_noalloc(const void* Q, const void* K, const void* V, const void* O, const void* dO, const float* LSE,
                   void* dQ, void* dK, void* dV, int B, int H, int N, int d, float scale, int causal, void* stream) {
  bool empty = false;
  const int rc0 = check_shape(B, H, H, N, N, d, scale, causal, &empty);
  if (rc0 != FA_OK) return rc0;
  if (!empty && fa_bwd_workspace_size(B, H, N, d) > FA_BWD_NOALLOC_SCRATCH_BYTES) return FA_ERR_UNSUPPORTED;
  int rc = FA_OK;
  void* ws = noalloc_scratch(&rc);
  if (!ws) return rc;
  // fa_bwd's preprocess kernel rewrites D and LSE*log2(e) and zeroes the dQ accumulator on every call.
  return fa_bwd(Q, K, V, O, dO, LSE, dQ, dK, dV, ws, FA_BWD_NOALLOC_SCRATCH_BYTES, B, H, N, d, scale, causal,
                stream);
}

int fa_last_device_status(void* stream, int* detail) {
  if (detail) *detail = 0;
  int rc = FA_OK;
  int* status = device_status(&rc);
  if (!status) return rc;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(status, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FA_ERR_CUDA;
    if (detail) *detail = v;
    return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}

unsigned elementwise_grid(long long items) {
  const long long blocks = (items + 255) / 256;
  return static_cast<unsigned>(blocks < 148 * 16 ? (blocks > 0 ? blocks : 1) : 148 * 16);
}

int fa_lse_merge(const void* O_part, const float* LSE_part, float* O_acc, float* LSE_acc, int64_t rows, int d,
                 int first, void* stream) {
  if (rows < 0 || (first != 0 && first != 1)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (rows == 0) return FA_OK;
  if (!O_part || !LSE_part || !O_acc || !LSE_acc) return FA_ERR_INVALID_ARG;
  if (!aligned16(O_part) || !aligned16(O_acc) || (reinterpret_cast<uintptr_t>(LSE_part) & 3u) ||
      (reinterpret_cast<uintptr_t>(LSE_acc) & 3u))
    return FA_ERR_ALIGNMENT;
  if (rows > (1LL << 40) / d) return FA_ERR_UNSUPPORTED;
  const size_t pb = static_cast<size_t>(rows) * d * 2, ab = static_cast<size_t>(rows) * d * 4, lb = rows * 4;
  if (overlaps(O_acc, ab, O_part, pb) || overlaps(O_acc, ab, LSE_part, lb) || overlaps(LSE_acc, lb, O_part, pb) ||
      overlaps(LSE_acc, lb, LSE_part, lb) || overlaps(O_acc, ab, LSE_acc, lb))
    return FA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const unsigned grid = elementwise_grid(rows * (d / 8));
  if (d == 128)
    fa::lse_merge_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(O_part), LSE_part, O_acc,
                                                    LSE_acc, rows, first);
  else
    fa::lse_merge_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(O_part), LSE_part, O_acc,
                                                   LSE_acc, rows, first);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_accumulate_bf16(float* acc, const void* x, int64_t n, int first, void* stream) {
  if (n < 0 || (n & 7) || (first != 0 && first != 1)) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!acc || !x) return FA_ERR_INVALID_ARG;
  if (!aligned16(acc) || !aligned16(x)) return FA_ERR_ALIGNMENT;
  if (overlaps(acc, static_cast<size_t>(n) * 4, x, static_cast<size_t>(n) * 2)) return FA_ERR_INVALID_ARG;
  fa::accumulate_bf16_kernel<<<elementwise_grid(n / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      acc, static_cast<const __nv_bfloat16*>(x), n / 8, first);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_accumulate_f32(float* acc, const float* x, int64_t n, void* stream) {
  if (n < 0 || (n & 7)) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!acc || !x) return FA_ERR_INVALID_ARG;
  if (!aligned16(acc) || !aligned16(x)) return FA_ERR_ALIGNMENT;
  if (overlaps(acc, static_cast<size_t>(n) * 4, x, static_cast<size_t>(n) * 4)) return FA_ERR_INVALID_ARG;
  fa::accumulate_f32_kernel<<<elementwise_grid(n / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(acc, x, n / 8);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_convert_f32_bf16(const float* x, void* y, int64_t n, void* stream) {
  if (n < 0 || (n & 7)) return FA_ERR_INVALID_ARG;
  if (n == 0) return FA_OK;
  if (!x || !y) return FA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return FA_ERR_ALIGNMENT;
  if (overlaps(x, static_cast<size_t>(n) * 4, y, static_cast<size_t>(n) * 2)) return FA_ERR_INVALID_ARG;
  fa::convert_f32_bf16_kernel<<<elementwise_grid(n / 8), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      x, static_cast<__nv_bfloat16*>(y), n / 8);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_set_forward_variant(int cluster_pair) {
  if (cluster_pair != 0 && cluster_pair != 1) return FA_ERR_INVALID_ARG;
  g_fwd_pair = cluster_pair;
  return FA_OK;
}

int fa_set_backward_variant(int cluster_pair) {
  if (cluster_pair != 0 && cluster_pair != 1) return FA_ERR_INVALID_ARG;
  g_bwd_pair = cluster_pair;
  return FA_OK;
}

int fa_profile_next(int which, void* start_event, void* stop_event) {
  if ((which != 0 && which != 1) || (!start_event) != (!stop_event)) return FA_ERR_INVALID_ARG;
  g_prof[which][0] = static_cast<cudaEvent_t>(start_event);
  g_prof[which][1] = static_cast<cudaEvent_t>(stop_event);
  return FA_OK;
}

int fa_sm_clock_probe(uint64_t* out, void* stream) {
  if (!out) return FA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(out) & 7u) return FA_ERR_ALIGNMENT;
  clock_probe_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(reinterpret_cast<unsigned long long*>(out));
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_selftest_wait_timeout(void* stream) {
  int rc = FA_OK;
  int* status = device_status(&rc);
  if (!status) return rc;
  selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(status);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_exp2_eval(const float* x, float* y, int64_t n, int mode, void* stream) {
  if (!x || !y || n < 0 || mode < 0 || mode > 2) return FA_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(y)) return FA_ERR_ALIGNMENT;
  if (n == 0) return FA_OK;
  if (n > (1LL << 36)) return FA_ERR_UNSUPPORTED;
  const unsigned grid = static_cast<unsigned>((n + 255) / 256);
  exp2_eval_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n, mode);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // extern "C"
