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

// Share of prefetch ranges taken by one of `parts` cooperating CTAs: each
// range is cut into `parts` 16-byte-aligned slices, and the slice of part
// `part` is issued in chunks of up to 32 KB by `nthr` threads (thread
// index `t`).
template <int NR>
__device__ __forceinline__ void l2_prefetch_share(const void* const (&p)[NR],
                                                  const long (&bytes)[NR],
                                                  int part, int parts, int t,
                                                  int nthr) {
  constexpr long kChunk = 32768;
#pragma unroll
  for (int r = 0; r < NR; ++r) {
    if (!p[r] || bytes[r] <= 0) continue;
    const long per = ((bytes[r] + parts - 1) / parts + 15) & ~15L;
    const long lo = (long)part * per;
    const long hi = lo + per < bytes[r] ? lo + per : bytes[r];
    for (long off = lo + (long)t * kChunk; off < hi; off += (long)nthr * kChunk) {
      const long n = hi - off < kChunk ? hi - off : kChunk;
      prefetch_l2(static_cast<const char*>(p[r]) + off, (uint32_t)n);
    }
  }
}

__device__ __forceinline__ float sigmoidf_(float x) {
  return 1.f / (1.f + __expf(-x));
}

// Sum of NV values over the whole block; every thread gets the results.
// `red` needs NV * (blockDim.x / 32) floats.  Contains __syncthreads().
template <int NV>
__device__ __forceinline__ void block_sum_n(float (&v)[NV], float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int nw = (blockDim.x + 31) >> 5;
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = warp_sum(v[i]);
  __syncthreads();
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NV; ++i) red[w * NV + i] = v[i];
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    float t = 0.f;
    for (int k = 0; k < nw; ++k) t += red[k * NV + i];
    v[i] = t;
  }
}

// nGPT residual update of one row held by the whole block:
//   s_new = N(s + alpha (N(h) - s)) = N((1 - alpha) s + alpha h / |h|),
//   h = sum of hS partials (stride h_stride).
// Both norms come from one block reduction: with a = 1 - alpha,
//   |t|^2 = sum (a s)^2 + 2 sum a alpha s h / |h| + sum (alpha h)^2 / |h|^2.
// Loop re-injection: RJ_FIRST stores x := s_new (x_row, if given) and
// returns N(s_new + x) = N(2 s_new) = s_new; RJ_NEXT returns
// N(s_new + x) using |s_new + x|^2 = 1 + 2 s_new.x + |x|^2, whose terms are
// reduced in the same pass.  Writes the result to dst (f32) and/or dst_bf
// (bf16) when non-null.  tmp holds d floats; red needs 7 * blockDim/32
// floats.  All threads must call it; it ends with __syncthreads().
__device__ inline void ngpt_update_row(const float* s, const float* h, int hS,
                                       size_t h_stride, const float* alpha,
                                       int d, int reinject, float* x_row,
                                       float* dst, bf16* dst_bf, float* tmp,
                                       float* red) {
  constexpr int U = 10;              // elements per thread in flight
  const int nt = blockDim.x;
  float r[7] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  const bool next = reinject == RJ_NEXT;
  for (int i0 = threadIdx.x; i0 < d; i0 += U * nt) {
    float hv[U], sv[U], av[U], xv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * nt;
      hv[u] = sv[u] = av[u] = xv[u] = 0.f;
      if (i < d) {
        sv[u] = s[i];
        av[u] = alpha[i];
        if (next) xv[u] = x_row[i];
      }
    }
#pragma unroll 4
    for (int k = 0; k < hS; ++k) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int i = i0 + u * nt;
        if (i < d) hv[u] += h[k * h_stride + i];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * nt;
      if (i < d) {
        tmp[i] = hv[u];
        const float as = (1.f - av[u]) * sv[u], ah = av[u] * hv[u];
        r[0] += hv[u] * hv[u];
        r[1] += as * as;
        r[2] += as * ah;
        r[3] += ah * ah;
        r[4] += as * xv[u];
        r[5] += ah * xv[u];
        r[6] += xv[u] * xv[u];
      }
    }
  }
  if (next) block_sum_n<7>(r, red);
  else {
    float q[4] = {r[0], r[1], r[2], r[3]};
    block_sum_n<4>(q, red);
    r[0] = q[0]; r[1] = q[1]; r[2] = q[2]; r[3] = q[3];
  }
  const float inv_h = 1.f / fmaxf(sqrtf(r[0]), 1e-12f);
  const float tt = r[1] + 2.f * r[2] * inv_h + r[3] * inv_h * inv_h;
  const float inv_t = 1.f / fmaxf(sqrtf(fmaxf(tt, 0.f)), 1e-12f);
  float inv_u = 1.f;
  if (next) {
    const float dot = (r[4] + r[5] * inv_h) * inv_t;
    inv_u = 1.f / fmaxf(sqrtf(fmaxf(1.f + 2.f * dot + r[6], 0.f)), 1e-12f);
  }
  for (int i0 = threadIdx.x; i0 < d; i0 += U * nt) {
    float sv[U], av[U], xv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * nt;
      sv[u] = av[u] = xv[u] = 0.f;
      if (i < d) {
        sv[u] = s[i];
        av[u] = alpha[i];
        if (next) xv[u] = x_row[i];
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = i0 + u * nt;
      if (i < d) {
        float v = ((1.f - av[u]) * sv[u] + av[u] * tmp[i] * inv_h) * inv_t;
        if (reinject == RJ_FIRST && x_row) x_row[i] = v;
        if (next) v = (v + xv[u]) * inv_u;
        if (dst) dst[i] = v;
        if (dst_bf) dst_bf[i] = __float2bfloat16_rn(v);
      }
    }
  }
  __syncthreads();
}

}  // namespace dory
