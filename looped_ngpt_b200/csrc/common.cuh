// Small device helpers shared by the kernels.
#pragma once
#include "dory_internal.h"

namespace dory {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1)
    v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Sum over the whole block; every thread gets the result.  `red` needs
// blockDim.x / 32 floats of shared memory.  Contains __syncthreads().
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

// BF16 pair held in a 32-bit word -> two floats (exact widening).
__device__ __forceinline__ float bf_lo(uint32_t u) {
  return __uint_as_float(u << 16);
}
__device__ __forceinline__ float bf_hi(uint32_t u) {
  return __uint_as_float(u & 0xffff0000u);
}

// 16-byte streaming load of weights: read once, do not keep in L1.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// Programmatic dependent launch.  Every kernel of the forward pass is
// launched so that it may start while its predecessor is still running.
// Rule used throughout: before pdl_wait() a kernel touches only immutable
// data (weights) or data written by kernels that finished before its
// predecessor started; it calls pdl_trigger() only after pdl_wait(), so at
// most one kernel runs ahead of the one it depends on.  Both are no-ops when
// the kernel was launched without the attribute.
__device__ __forceinline__ void pdl_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Ask L2 to start fetching [p, p + bytes) (no data returned).  p and bytes
// must be multiples of 16.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  if (bytes == 0) return;
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ float sigmoidf_(float x) {
  return 1.f / (1.f + __expf(-x));
}

// nGPT residual update of one row held by the whole block:
//   s_new = N(s + alpha (N(h) - s)),  h = sum of h_S partials.
// Optional loop re-injection: RJ_FIRST stores x := s_new and returns
// N(s_new + x); RJ_NEXT returns N(s_new + x) with the stored x.
// dst receives the row (f32) when non-null; dst_bf (bf16) likewise.
// `red` needs blockDim/32 floats.  All threads must call it.
__device__ inline void ngpt_update_row(const float* s, const float* h, int hS,
                                       size_t h_stride, const float* alpha,
                                       int d, int reinject, float* x_row,
                                       float* dst, bf16* dst_bf, float* tmp,
                                       float* red) {
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float v = 0.f;
    for (int k = 0; k < hS; ++k) v += h[k * h_stride + i];
    tmp[i] = v;
    ss += v * v;
  }
  const float inv_h = 1.f / fmaxf(sqrtf(block_sum(ss, red)), 1e-12f);
  float tt = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float sv = s[i];
    float t = sv + alpha[i] * (tmp[i] * inv_h - sv);
    tmp[i] = t;
    tt += t * t;
  }
  const float inv_t = 1.f / fmaxf(sqrtf(block_sum(tt, red)), 1e-12f);
  if (reinject == RJ_NONE) {
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
      float v = tmp[i] * inv_t;
      tmp[i] = v;
      if (dst) dst[i] = v;
      if (dst_bf) dst_bf[i] = __float2bfloat16_rn(v);
    }
    __syncthreads();
    return;
  }
  float uu = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float v = tmp[i] * inv_t;
    float xv;
    if (reinject == RJ_FIRST) {
      xv = v;
      if (x_row) x_row[i] = v;
    } else {
      xv = x_row[i];
    }
    float u = v + xv;
    tmp[i] = u;
    uu += u * u;
  }
  const float inv_u = 1.f / fmaxf(sqrtf(block_sum(uu, red)), 1e-12f);
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    float v = tmp[i] * inv_u;
    tmp[i] = v;
    if (dst) dst[i] = v;
    if (dst_bf) dst_bf[i] = __float2bfloat16_rn(v);
  }
  __syncthreads();
}

}  // namespace dory
