// fa_merge.cuh -- combining attention results over disjoint key sets, and the fp32
// accumulation helpers of the ring (context-parallel) driver.
//
// Exact attention over the union of disjoint key sets follows from the results over each set:
// with L = ln(exp(LSE_a) + exp(LSE_b)),  O = exp(LSE_a - L) O_a + exp(LSE_b - L) O_b.  This is the
// per-row log-sum-exp that the forward returns, used the way the online softmax combines key tiles
// ("The Technical Edge", adaptive online softmax rescaling), one level up: the pages name context /
// multi-card parallelism for long sequences ("NVIDIA Blackwell: FlashAttention-4 Overcomes Memory
// Bottlenecks", body).  All three kernels are HBM-bound elementwise passes: 16-byte vector
// accesses, grid-stride loops.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace fa {

// One thread per 8 elements (16 bytes of bf16) of a row of d (64 or 128) columns.  The G threads
// of a row are consecutive lanes of one warp; each reads the row's old LSE, and the row's last
// lane writes the new one after a __syncwarp, so no lane can read the new value.  Every thread of
// the block runs the same number of loop iterations (the stride is uniform), as __syncwarp needs.
template <int D>
__global__ void __launch_bounds__(256) lse_merge_kernel(const __nv_bfloat16* __restrict__ o_part,
                                                        const float* __restrict__ lse_part, float* __restrict__ o_acc,
                                                        float* __restrict__ lse_acc, long long rows, int first) {
  constexpr int G = D / 8;
  const long long total = rows * G;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long t0 = static_cast<long long>(blockIdx.x) * blockDim.x; t0 < total; t0 += stride) {
    const long long t = t0 + threadIdx.x;
    const bool live = t < total;
    const long long r = live ? t / G : 0;
    const int seg = static_cast<int>(t % G);
    float lnew = 0.0f;
    if (live) {
      const float lp = lse_part[r];
      const uint4 raw = *reinterpret_cast<const uint4*>(o_part + r * D + seg * 8);
      const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&raw);
      float4* acc = reinterpret_cast<float4*>(o_acc + r * D + seg * 8);
      float wa = 0.0f, wp = 1.0f;
      lnew = lp;
      float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
      if (!first) {
        const float la = lse_acc[r];
        const float m = fmaxf(la, lp);
        if (m == -INFINITY) {  // no key seen on either side
          wa = wp = 0.0f;
          lnew = -INFINITY;
        } else {
          const float ea = expf(la - m), ep = expf(lp - m);
          const float s = ea + ep;
          wa = ea / s;
          wp = ep / s;
          lnew = m + logf(s);
        }
        a0 = acc[0];
        a1 = acc[1];
      }
      const float2 p0 = __bfloat1622float2(pb[0]), p1 = __bfloat1622float2(pb[1]);
      const float2 p2 = __bfloat1622float2(pb[2]), p3 = __bfloat1622float2(pb[3]);
      acc[0] = make_float4(wa * a0.x + wp * p0.x, wa * a0.y + wp * p0.y, wa * a0.z + wp * p1.x, wa * a0.w + wp * p1.y);
      acc[1] = make_float4(wa * a1.x + wp * p2.x, wa * a1.y + wp * p2.y, wa * a1.z + wp * p3.x, wa * a1.w + wp * p3.y);
    }
    __syncwarp();
    if (live && seg == G - 1) lse_acc[r] = lnew;
  }
}

// acc (fp32, n) = (first ? 0 : acc) + x (bf16, n); n a multiple of 8.
__global__ void __launch_bounds__(256) accumulate_bf16_kernel(float* __restrict__ acc,
                                                              const __nv_bfloat16* __restrict__ x, long long n8,
                                                              int first) {
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < n8;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 raw = *reinterpret_cast<const uint4*>(x + t * 8);
    const __nv_bfloat162* pb = reinterpret_cast<const __nv_bfloat162*>(&raw);
    float4* a = reinterpret_cast<float4*>(acc + t * 8);
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
    if (!first) {
      a0 = a[0];
      a1 = a[1];
    }
    const float2 p0 = __bfloat1622float2(pb[0]), p1 = __bfloat1622float2(pb[1]);
    const float2 p2 = __bfloat1622float2(pb[2]), p3 = __bfloat1622float2(pb[3]);
    a[0] = make_float4(a0.x + p0.x, a0.y + p0.y, a0.z + p1.x, a0.w + p1.y);
    a[1] = make_float4(a1.x + p2.x, a1.y + p2.y, a1.z + p3.x, a1.w + p3.y);
  }
}

// acc (fp32, n) += x (fp32, n); n a multiple of 8.
__global__ void __launch_bounds__(256) accumulate_f32_kernel(float* __restrict__ acc, const float* __restrict__ x,
                                                             long long n8) {
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < n8;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(x + t * 8);
    float4* a = reinterpret_cast<float4*>(acc + t * 8);
    const float4 x0 = src[0], x1 = src[1];
    float4 a0 = a[0], a1 = a[1];
    a[0] = make_float4(a0.x + x0.x, a0.y + x0.y, a0.z + x0.z, a0.w + x0.w);
    a[1] = make_float4(a1.x + x1.x, a1.y + x1.y, a1.z + x1.z, a1.w + x1.w);
  }
}

// y (bf16, n) = round-to-nearest-even(x (fp32, n)); n a multiple of 8.
__global__ void __launch_bounds__(256) convert_f32_bf16_kernel(const float* __restrict__ x,
                                                               __nv_bfloat16* __restrict__ y, long long n8) {
  for (long long t = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; t < n8;
       t += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4* src = reinterpret_cast<const float4*>(x + t * 8);
    const float4 a = src[0], b = src[1];
    __nv_bfloat162 o[4] = {__floats2bfloat162_rn(a.x, a.y), __floats2bfloat162_rn(a.z, a.w),
                           __floats2bfloat162_rn(b.x, b.y), __floats2bfloat162_rn(b.z, b.w)};
    *reinterpret_cast<uint4*>(y + t * 8) = *reinterpret_cast<const uint4*>(o);
  }
}

}  // namespace fa
