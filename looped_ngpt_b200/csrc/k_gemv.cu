// Weight-streaming GEMV for small-batch decode (B <= 8 rows of activations):
// y[b][n] = sum_k W[n][k] x[b][k], W bf16 row-major, read exactly once.
//
// Blackwell design: one block per SM owns a contiguous range of work items
// (an output row, or a 2560-wide K segment of one for long rows; a gate/up
// row pair for SwiGLU), i.e. one contiguous byte range of W (two for the
// pair).  A producer warp streams that range through a ring of NS
// shared-memory stages of 8 items with 1-D TMA bulk copies
// (cp.async.bulk ... mbarrier::complete_tx), so 80-160 KB per SM are in
// flight without spending registers.  Each of the 8 consumer warps owns one
// item of every stage, reduces it with shuffles, writes its output and
// releases the stage on an "empty" mbarrier: there is no block-wide barrier
// in the streaming loop.  The first stages are issued before
// the programmatic-dependent-launch wait: the weights do not depend on the
// previous kernel, so HBM starts streaming while the predecessor finishes and
// while this kernel's prologue runs.  Every mbarrier wait is bounded; on
// timeout the block records ERRBIT_TIMEOUT, waits (bounded) for the copies it
// issued and exits.
//
// Prologue PRO_UPDATE fuses the previous sublayer's nGPT residual update
// (s <- N(s + alpha (N(h) - s)), "Dory1.0-4B: A Looped Normalized-GPT" §2)
// and the loop-boundary re-injection u_t = N(s_{t-1} + x) (paper summary,
// 核心方法): every block recomputes the d-length update from L2-resident
// vectors and block 0 writes the new state, so no separate launch or
// grid-wide synchronisation is needed.
//
// Epilogues: EPI_F32 (plain), EPI_SWIGLU (rows n and n + F of the fused
// gate/up matrix -> silu(gate) * up as bf16; the L2 norm that precedes the
// down projection is dropped because the normalised update makes it a
// no-op: N(W N(m)) = N(W m)), EPI_LMHEAD (logit scale s_z, optional logits
// store, per-block greedy argmax partials).
#include <cstdlib>

#include <cuda_fp16.h>

#include "common.cuh"

namespace dory {

namespace {

constexpr int kWarps = 8;                    // consumer warps
constexpr int kThreads = (kWarps + 1) * 32;  // + one producer warp
constexpr int kMaxStages = 8;
constexpr int kSeg = 2560;                   // max K segment per item
constexpr long kSpinLimit = 1L << 26;   // bounded mbarrier polls

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar))
               : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(
          smem_addr(bar)),
      "r"(bytes)
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n"
      " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  for (long i = 0; i < kSpinLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

__device__ __forceinline__ void tma_load_1d(void* dst, const void* src,
                                            uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

struct Plan {
  int S;        // K segments per row (items per row)
  int NS;       // stages in the ring (8 items each)
};

// ---- quantised weights (MXFP8 / NVFP4): decode 8 weights of one lane ----
__device__ __forceinline__ float2 half2_to_float2(uint32_t h) {
  __half2 v = *reinterpret_cast<__half2*>(&h);
  return __half22float2(v);
}
// E4M3 pair (low byte first) -> two floats, exact (via f16).
__device__ __forceinline__ float2 e4m3x2_f2(uint16_t v) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(v));
  return half2_to_float2(h);
}
// E2M1 pair (low nibble first) -> two floats, exact (via f16).
__device__ __forceinline__ float2 e2m1x2_f2(uint32_t byte) {
  uint32_t h;
  asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }"
      : "=r"(h)
      : "r"(byte));
  return half2_to_float2(h);
}
// E8M0 scale 2^(e - 127); code 0 is 2^-127 (an f32 subnormal), 0xFF NaN.
__device__ __forceinline__ float e8m0_f(uint32_t e) {
  return e == 0 ? __uint_as_float(0x00400000u)
                : (e == 255 ? __uint_as_float(0x7fc00000u) : __uint_as_float(e << 23));
}
__device__ __forceinline__ float e4m3_f(uint32_t b) {
  return e4m3x2_f2((uint16_t)(b & 0xFF)).x;
}

// Bytes of one lane's 8 weights, and weights per scale.
template <int FMT> struct FmtInfo;
template <> struct FmtInfo<WF_BF16> { static constexpr int LB = 16, GROUP = 0; };
template <> struct FmtInfo<WF_MXFP8> { static constexpr int LB = 8, GROUP = 32; };
template <> struct FmtInfo<WF_NVFP4> { static constexpr int LB = 4, GROUP = 16; };

template <int FMT>
__device__ __forceinline__ void decode8(const uint8_t* p, float (&w)[8]) {
  if (FMT == WF_BF16) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    w[0] = bf_lo(v.x); w[1] = bf_hi(v.x); w[2] = bf_lo(v.y); w[3] = bf_hi(v.y);
    w[4] = bf_lo(v.z); w[5] = bf_hi(v.z); w[6] = bf_lo(v.w); w[7] = bf_hi(v.w);
  } else if (FMT == WF_MXFP8) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    float2 f;
    f = e4m3x2_f2((uint16_t)(v.x & 0xFFFF)); w[0] = f.x; w[1] = f.y;
    f = e4m3x2_f2((uint16_t)(v.x >> 16)); w[2] = f.x; w[3] = f.y;
    f = e4m3x2_f2((uint16_t)(v.y & 0xFFFF)); w[4] = f.x; w[5] = f.y;
    f = e4m3x2_f2((uint16_t)(v.y >> 16)); w[6] = f.x; w[7] = f.y;
  } else {
    const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
    float2 f;
    f = e2m1x2_f2(v & 0xFF); w[0] = f.x; w[1] = f.y;
    f = e2m1x2_f2((v >> 8) & 0xFF); w[2] = f.x; w[3] = f.y;
    f = e2m1x2_f2((v >> 16) & 0xFF); w[4] = f.x; w[5] = f.y;
    f = e2m1x2_f2(v >> 24); w[6] = f.x; w[7] = f.y;
  }
}

// Scale of the group holding element k of row `row` (1.f for BF16).
template <int FMT>
__device__ __forceinline__ float group_scale(const uint8_t* Ws, int K, long row,
                                             int k) {
  if (FMT == WF_MXFP8) return e8m0_f(__ldg(Ws + row * (K / 32) + k / 32));
  if (FMT == WF_NVFP4) return e4m3_f(__ldg(Ws + row * (K / 16) + k / 16));
  return 1.f;
}

// One staged row segment (item) times the register-resident x slice
// (batch 1).  Lane covers elements c * 256 + lane * 8 + [0, 8), c < nc; its
// 8 weights share one group scale (groups of 32 / 16 elements).
template <int FMT, int MAXC>
__device__ __forceinline__ float row_dot_reg_q(const uint8_t* wb, const float* xr,
                                               const float* scl, int nc,
                                               int lane) {
  constexpr int LB = FmtInfo<FMT>::LB;
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    if (c < nc) {
      float w[8];
      decode8<FMT>(wb + (c * 32 + lane) * LB, w);
      float t0 = w[0] * xr[c * 8 + 0], t1 = w[1] * xr[c * 8 + 1];
      t0 = fmaf(w[2], xr[c * 8 + 2], t0); t1 = fmaf(w[3], xr[c * 8 + 3], t1);
      t0 = fmaf(w[4], xr[c * 8 + 4], t0); t1 = fmaf(w[5], xr[c * 8 + 5], t1);
      t0 = fmaf(w[6], xr[c * 8 + 6], t0); t1 = fmaf(w[7], xr[c * 8 + 7], t1);
      if (FMT == WF_BF16) { a0 += t0; a1 += t1; }
      else { a0 = fmaf(t0, scl[c], a0); a1 = fmaf(t1, scl[c], a1); }
    }
  }
  return warp_sum(a0 + a1);
}

// Batched variant: x from shared memory (bf16 [NB][K], slice at xk).
template <int FMT, int NB, int MAXC>
__device__ __forceinline__ void row_dot_smem_q(const uint8_t* wb, const bf16* xk,
                                               int K, const float* scl, int nc,
                                               int lane, float (&acc)[NB]) {
  constexpr int LB = FmtInfo<FMT>::LB;
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = 0.f;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    if (c < nc) {
      float w[8];
      decode8<FMT>(wb + (c * 32 + lane) * LB, w);
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        const uint4 xv = *reinterpret_cast<const uint4*>(xk + b * K + c * 256 + lane * 8);
        float t = w[0] * bf_lo(xv.x);
        t = fmaf(w[1], bf_hi(xv.x), t); t = fmaf(w[2], bf_lo(xv.y), t);
        t = fmaf(w[3], bf_hi(xv.y), t); t = fmaf(w[4], bf_lo(xv.z), t);
        t = fmaf(w[5], bf_hi(xv.z), t); t = fmaf(w[6], bf_lo(xv.w), t);
        t = fmaf(w[7], bf_hi(xv.w), t);
        acc[b] = FMT == WF_BF16 ? acc[b] + t : fmaf(t, scl[c], acc[b]);
      }
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
}

// Activation vector(s) for the GEMV -> shared memory as bf16: a copy of the
// caller's bf16 rows (PRO_BF16) or the fused nGPT update (PRO_UPDATE).
template <int NB>
__device__ __forceinline__ void gemv_prologue(const GemvArgs& a, bf16* xs,
                                              float* tmp, float* red) {
  const int K = a.K, tid = threadIdx.x;
  if (a.pro == PRO_BF16) {
    const int vec = K / 8;
    for (int b = 0; b < NB; ++b) {
      uint4* dst = reinterpret_cast<uint4*>(xs + b * K);
      if (b < a.B) {
        const uint4* src =
            reinterpret_cast<const uint4*>(a.xin + (size_t)b * a.xin_stride);
        for (int i = tid; i < vec; i += kThreads) dst[i] = src[i];
      } else {
        for (int i = tid; i < vec; i += kThreads) dst[i] = make_uint4(0, 0, 0, 0);
      }
    }
  } else {
    for (int b = 0; b < NB; ++b) {
      if (b < a.B) {
        float* xrow = nullptr;
        if (a.reinject == RJ_FIRST && blockIdx.x == 0) xrow = a.x_buf + b * K;
        if (a.reinject == RJ_NEXT) xrow = a.x_buf + b * K;
        ngpt_update_row(a.s_in + (size_t)b * K, a.h_in + (size_t)b * K,
                        a.h_S, (size_t)a.B * K, a.alpha, K, a.reinject, xrow,
                        blockIdx.x == 0 ? a.s_out + (size_t)b * K : nullptr,
                        xs + b * K, tmp, red);
      } else {
        for (int i = tid; i < K; i += kThreads)
          xs[b * K + i] = __float2bfloat16_rn(0.f);
      }
    }
  }
  __syncthreads();
}


template <int NB, int EPI, int FMT>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(const GemvArgs a, const Plan pl) {
  constexpr int R = (EPI == EPI_SWIGLU) ? 2 : 1;
  constexpr int LB = FmtInfo<FMT>::LB;       // bytes per 8 weights
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = a.K, S = pl.S, NS = pl.NS;
  const int seg = K / S;
  const size_t item_bytes = (size_t)seg / 8 * LB;
  const size_t stage_bytes = (size_t)kWarps * R * item_bytes;
  uint8_t* ring = smem;                                         // NS stages
  bf16* xs = reinterpret_cast<bf16*>(ring + NS * stage_bytes);  // [NB][K]
  float* tmp = reinterpret_cast<float*>(xs + NB * K);           // [K] if UPDATE
  uint64_t* full = reinterpret_cast<uint64_t*>(
      tmp + (a.pro == PRO_UPDATE ? K : 0));
  uint64_t* empty = full + NS;
  __shared__ float red[7 * (kWarps + 1)];
  __shared__ float bestv[kWarps][NB];
  __shared__ int besti[kWarps][NB];
  __shared__ int s_fail, s_issued;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // row-aligned item range: a stage of 8 items starts at a multiple of S,
  // so warp w always works on K segment w % S
  const long j0 = (long)a.n_items * blockIdx.x / gridDim.x * S;
  const long j1 = (long)a.n_items * (blockIdx.x + 1) / gridDim.x * S;
  const int n_stages = (int)((j1 - j0 + kWarps - 1) / kWarps);
  const bool producer = tid == kWarps * 32;

  // items j0.. are contiguous in W: item it = (row it / S, segment it % S)
  auto issue = [&](int s) {
    const long it = j0 + (long)s * kWarps;
    const long cnt = j1 - it < kWarps ? j1 - it : kWarps;
    const uint32_t bytes = (uint32_t)(cnt * item_bytes);
    uint64_t* bar = full + (s % NS);
    uint8_t* dst = ring + (s % NS) * stage_bytes;
    const char* w = FMT == WF_BF16 ? reinterpret_cast<const char*>(a.W)
                                   : reinterpret_cast<const char*>(a.Wq);
    mbar_expect_tx(bar, bytes * R);
    tma_load_1d(dst, w + it * item_bytes, bytes, bar);
    if (R == 2)
      tma_load_1d(dst + kWarps * item_bytes,
                  w + (it + (long)a.pair_off * S) * item_bytes, bytes, bar);
  };

  if (producer) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_fail = 0;
    const int n0 = NS < n_stages ? NS : n_stages;
    for (int s = 0; s < n0; ++s) issue(s);      // weights only: before the wait
    s_issued = n0;
  }
  pdl_wait();
  pdl_trigger();
  gemv_prologue<NB>(a, xs, tmp, red);           // ends with __syncthreads()

  volatile int* fail = &s_fail;
  float bv[NB];
  int bi[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) { bv[b] = -INFINITY; bi[b] = 0x7fffffff; }

  if (warp == kWarps) {
    // ---- producer: refill a slot once all consumer warps released it ----
    if (lane == 0) {
      for (int s = NS; s < n_stages && !*fail; ++s) {
        const int slot = s % NS, use = s / NS;
        if (!mbar_wait(empty + slot, (uint32_t)((use - 1) & 1))) {
          atomicOr(&s_fail, 1);
          break;
        }
        issue(s);
        s_issued = s + 1;
      }
    }
  } else {
    // ---- consumers: warp w owns item w of every stage ------------------
    // NB == 1: this warp's slice of x (segment w % S, lane's 8-element
    // chunks) stays in registers as f32 for the whole kernel.
    constexpr int kMaxC = kSeg / 256;
    const int nc = seg >> 8;
    float xr[NB == 1 ? kMaxC * 8 : 1];
    if (NB == 1) {
      const bf16* xk = xs + (warp % S) * seg + lane * 8;
#pragma unroll
      for (int c = 0; c < kMaxC; ++c) {
        if (c < nc) {
          const uint4 xv = *reinterpret_cast<const uint4*>(xk + c * 256);
          xr[c * 8 + 0] = bf_lo(xv.x); xr[c * 8 + 1] = bf_hi(xv.x);
          xr[c * 8 + 2] = bf_lo(xv.y); xr[c * 8 + 3] = bf_hi(xv.y);
          xr[c * 8 + 4] = bf_lo(xv.z); xr[c * 8 + 5] = bf_hi(xv.z);
          xr[c * 8 + 6] = bf_lo(xv.w); xr[c * 8 + 7] = bf_hi(xv.w);
        }
      }
    }
    for (int s = 0; s < n_stages; ++s) {
      const int slot = s % NS;
      const long it = j0 + (long)s * kWarps + warp;
      const bool has = it < j1;
      const int n = has ? (int)(it / S) : 0;
      const int sidx = has ? (int)(it - (long)n * S) : 0;
      // group scales of this lane's chunks, fetched before the stage lands
      float sc1[FMT == WF_BF16 ? 1 : kMaxC], sc2[FMT == WF_BF16 ? 1 : kMaxC];
      if (FMT != WF_BF16 && has) {
#pragma unroll
        for (int c = 0; c < kMaxC; ++c) {
          if (c < nc) {
            const int k = sidx * seg + c * 256 + lane * 8;
            sc1[c] = group_scale<FMT>(a.Ws, K, n, k);
            if (R == 2) sc2[c] = group_scale<FMT>(a.Ws, K, (long)n + a.pair_off, k);
          }
        }
      }
      if (!mbar_wait(full + slot, (uint32_t)((s / NS) & 1))) {
        if (lane == 0) atomicOr(&s_fail, 1);
        break;
      }
      if (has) {
        float scl = 0.f;
        if (EPI == EPI_LMHEAD && lane == 0) scl = a.col_scale[n];
        const uint8_t* wb = ring + slot * stage_bytes + warp * item_bytes;
        float acc[NB], acc2[NB];
        if (NB == 1) {
          acc[0] = row_dot_reg_q<FMT, kMaxC>(wb, xr, sc1, nc, lane);
          if (R == 2)
            acc2[0] = row_dot_reg_q<FMT, kMaxC>(wb + kWarps * item_bytes, xr, sc2,
                                                nc, lane);
        } else {
          row_dot_smem_q<FMT, NB, kMaxC>(wb, xs + sidx * seg, K, sc1, nc, lane, acc);
          if (R == 2)
            row_dot_smem_q<FMT, NB, kMaxC>(wb + kWarps * item_bytes, xs, K, sc2,
                                           nc, lane, acc2);
        }
        if (FMT == WF_NVFP4) {            // per-tensor second-level scale
          const float ts = __ldg(a.Wt);
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            acc[b] *= ts;
            if (R == 2) acc2[b] *= ts;
          }
        }
        if (lane == 0) {
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if (b >= a.B) break;
            if (EPI == EPI_F32) {
              a.out[((size_t)sidx * a.B + b) * a.n_items + n] = acc[b];
            } else if (EPI == EPI_SWIGLU) {
              const float g = acc[b];
              a.out_bf[(size_t)b * a.pair_off + n] =
                  __float2bfloat16_rn(g * sigmoidf_(g) * acc2[b]);
            } else {
              const float z = scl * acc[b];
              if (a.out) a.out[(size_t)b * a.out_stride + n] = z;
              if (z > bv[b]) { bv[b] = z; bi[b] = n; }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + slot);
      if (*fail) break;
    }
  }
  __syncthreads();

  if (*fail) {
    // a bounded wait gave up: record it, wait (bounded) for the copies that
    // may still be landing in shared memory, then leave
    if (tid == 0) {
      atomicOr(a.err, ERRBIT_TIMEOUT);
      const int hi = s_issued, lo = hi - NS > 0 ? hi - NS : 0;
      for (int q = lo; q < hi; ++q)
        if (!mbar_wait(full + (q % NS), (uint32_t)((q / NS) & 1))) break;
    }
    return;
  }

  if (EPI == EPI_LMHEAD) {
    if (warp < kWarps && lane == 0) {
#pragma unroll
      for (int b = 0; b < NB; ++b) { bestv[warp][b] = bv[b]; besti[warp][b] = bi[b]; }
    }
    __syncthreads();
    if (tid < a.B && tid < NB) {
      float m = -INFINITY;
      int mi = 0x7fffffff;
      for (int q = 0; q < kWarps; ++q) {
        const float c = bestv[q][tid];
        const int ci = besti[q][tid];
        if (c > m || (c == m && ci < mi)) { m = c; mi = ci; }
      }
      a.amax_val[tid * gridDim.x + blockIdx.x] = m;
      a.amax_idx[tid * gridDim.x + blockIdx.x] = mi;
    }
  }
}

int stages_default() {
  static const int v = [] {
    const char* e = getenv("DORY_GEMV_STAGES");
    int n = e ? atoi(e) : 4;
    return n < 2 ? 2 : (n > kMaxStages ? kMaxStages : n);
  }();
  return v;
}

constexpr size_t kSmemBudget = 220 * 1024;

size_t fixed_smem(const GemvArgs& a, int nb) {
  return (size_t)nb * a.K * 2 + (a.pro == PRO_UPDATE ? (size_t)a.K * 4 : 0) +
         2 * kMaxStages * 8;
}

// Segments per row S (F32 only: SwiGLU and LM head need whole rows) and
// ring depth: the largest segment <= kSeg whose 8-item stages still fit at
// least 3 deep (2 as a last resort).
int lane_bytes(int fmt) { return fmt == WF_BF16 ? 16 : fmt == WF_MXFP8 ? 8 : 4; }

// Segments per row S (F32 only: SwiGLU and LM head need whole rows) and
// ring depth: the largest segment <= kSeg whose 8-item stages still fit at
// least 3 deep (2 as a last resort).
Plan make_plan(const GemvArgs& a, int nb) {
  const int R = a.epi == EPI_SWIGLU ? 2 : 1;
  const size_t fixed = fixed_smem(a, nb);
  const int lb = lane_bytes(a.fmt);
  int S = 1;
  if (a.epi == EPI_F32) {
    while (a.K / S > kSeg && (a.K / (2 * S)) % 256 == 0) S *= 2;
    while ((a.K / (2 * S)) % 256 == 0 &&
           fixed + 3 * (size_t)kWarps * R * (a.K / S) / 8 * lb > kSmemBudget)
      S *= 2;
  }
  const size_t stage = (size_t)kWarps * R * (a.K / S) / 8 * lb;
  int NS = stages_default();
  if (a.fmt != WF_BF16) NS = kMaxStages;          // smaller items: go deeper
  while (NS > 2 && fixed + NS * stage > kSmemBudget) --NS;
  return Plan{S, NS};
}

size_t smem_bytes(const GemvArgs& a, const Plan& p, int nb) {
  const int R = a.epi == EPI_SWIGLU ? 2 : 1;
  return (size_t)p.NS * kWarps * R * (a.K / p.S) / 8 * lane_bytes(a.fmt) +
         fixed_smem(a, nb);
}

int nb_of(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : 8; }

template <int NB, int EPI, int FMT>
void launch_t(const GemvArgs& a, int grid, cudaStream_t st) {
  const Plan pl = make_plan(a, NB);
  const size_t smem = smem_bytes(a, pl, NB);
  static size_t configured = 0;
  if (smem > configured) {
    cudaFuncSetAttribute(gemv_kernel<NB, EPI, FMT>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    configured = smem;
  }
  launch_k(gemv_kernel<NB, EPI, FMT>, dim3(grid), dim3(kThreads), smem, st, a,
           pl);
}

template <int NB, int EPI>
void launch_f(const GemvArgs& a, int grid, cudaStream_t st) {
  switch (a.fmt) {
    case WF_MXFP8: launch_t<NB, EPI, WF_MXFP8>(a, grid, st); break;
    case WF_NVFP4: launch_t<NB, EPI, WF_NVFP4>(a, grid, st); break;
    default: launch_t<NB, EPI, WF_BF16>(a, grid, st); break;
  }
}

template <int NB>
void launch_nb(const GemvArgs& a, int grid, cudaStream_t st) {
  switch (a.epi) {
    case EPI_F32: launch_f<NB, EPI_F32>(a, grid, st); break;
    case EPI_SWIGLU: launch_f<NB, EPI_SWIGLU>(a, grid, st); break;
    default: launch_t<NB, EPI_LMHEAD, WF_BF16>(a, grid, st); break;
  }
}

// Decode rows of a quantised matrix to f32 (tests: bit-exact against the
// format definitions); one thread per 8 consecutive weights.
template <int FMT>
__global__ void dequant_rows_kernel(const uint8_t* Wq, const uint8_t* Ws, int K,
                                    int row0, int nrows, float* out) {
  const long total = (long)nrows * K / 8;
  for (long id = blockIdx.x * (long)blockDim.x + threadIdx.x; id < total;
       id += (long)gridDim.x * blockDim.x) {
    const long r = id / (K / 8);
    const int k = (int)(id - r * (K / 8)) * 8;
    const long row = row0 + r;
    float w[8];
    decode8<FMT>(Wq + (row * K + k) / 8 * FmtInfo<FMT>::LB, w);
    const float sc = group_scale<FMT>(Ws, K, row, k);
#pragma unroll
    for (int e = 0; e < 8; ++e) out[r * K + k + e] = w[e] * sc;
  }
}

}  // namespace

int gemv_splits(const GemvArgs& a) { return make_plan(a, nb_of(a.B)).S; }

int gemv_grid(const GemvArgs& a, int num_sms) {
  return a.n_items < num_sms ? a.n_items : num_sms;
}

void launch_dequant_rows(int fmt, const uint8_t* Wq, const uint8_t* Ws, int K,
                         int row0, int nrows, float* out, cudaStream_t st) {
  if (fmt == WF_MXFP8)
    dequant_rows_kernel<WF_MXFP8><<<592, 256, 0, st>>>(Wq, Ws, K, row0, nrows, out);
  else
    dequant_rows_kernel<WF_NVFP4><<<592, 256, 0, st>>>(Wq, Ws, K, row0, nrows, out);
}

void launch_gemv(const GemvArgs& a, int grid, cudaStream_t st) {
  if (a.B <= 1) launch_nb<1>(a, grid, st);
  else if (a.B <= 2) launch_nb<2>(a, grid, st);
  else if (a.B <= 4) launch_nb<4>(a, grid, st);
  else launch_nb<8>(a, grid, st);
}

}  // namespace dory
