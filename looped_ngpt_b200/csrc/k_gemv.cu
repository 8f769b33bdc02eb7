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
// in the streaming loop.  The activations sit in shared memory and the
// per-lane K loop stays rolled, which keeps the loop body inside the
// instruction cache (a fully unrolled body with register-resident x was
// measured 2-3x slower per stage: its code was re-fetched every stage).  The first stages are issued before
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
// grid-wide synchronisation is needed.  Each thread holds its elements in
// registers across the block reduction (one L2 round trip; alpha is read
// before the dependent-launch wait).
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

// The same copy with an L2 eviction-priority hint: streamed weights are read
// once per call, and evict-first keeps them from displacing the small
// vectors (states, partial outputs, per-layer scales, KV tiles) that the
// dependent kernels read next.
__device__ __forceinline__ void tma_load_1d_hint(void* dst, const void* src,
                                                 uint32_t bytes, uint64_t* bar,
                                                 uint64_t pol) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

struct Plan {
  int S;        // K segments per row (items per row), a power of two
  int sh;       // log2(S)
  int NS;       // stages in the ring (8 items each)
  int tmp;      // PRO_UPDATE needs the two-pass prologue (K > kU * kThreads)
  int bps;      // blocks per SM (the grid is up to bps x the SM count)
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

// Bytes of one lane's 8 weights (scales cover 32 / 16 weights).
template <int FMT> struct FmtInfo;
template <> struct FmtInfo<WF_BF16> { static constexpr int LB = 16; };
template <> struct FmtInfo<WF_MXFP8> { static constexpr int LB = 8; };
template <> struct FmtInfo<WF_NVFP4> { static constexpr int LB = 4; };

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

// ---- consumer arithmetic ------------------------------------------------
// The streaming loop is kept compact on purpose: a fully unrolled K loop
// (x held in registers) made the loop body larger than the instruction cache
// and every stage re-fetched its code.  Here x lives in shared memory in the
// multiply format (bf16 for BF16 weights, f16 for the quantised formats) and
// a lane walks its 8-weight chunks c = lane, lane + 32, ... in a short
// rolled loop (two chunks per trip for ILP).

// Quantised codes of one lane chunk -> four exact f16 pairs (hardware cvt).
template <int FMT>
__device__ __forceinline__ void decode8_h2(const uint8_t* p, __half2 (&w)[4]) {
  if (FMT == WF_MXFP8) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    const uint16_t c[4] = {(uint16_t)(v.x & 0xFFFF), (uint16_t)(v.x >> 16),
                           (uint16_t)(v.y & 0xFFFF), (uint16_t)(v.y >> 16)};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t h;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c[i]));
      w[i] = *reinterpret_cast<__half2*>(&h);
    }
  } else {
    const uint32_t v = *reinterpret_cast<const uint32_t*>(p);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint32_t h;
      asm("{ .reg .b8 t; cvt.u8.u32 t, %1; cvt.rn.f16x2.e2m1x2 %0, t; }"
          : "=r"(h)
          : "r"((v >> (8 * i)) & 0xFF));
      w[i] = *reinterpret_cast<__half2*>(&h);
    }
  }
}

// 8-term dot product of decoded f16 weights with 8 f16 activations: packed
// f16 multiply-adds, the pair sum widened to f32.
__device__ __forceinline__ float dot8_h2(const __half2 (&w)[4], const uint4 xv) {
  const __half2* x = reinterpret_cast<const __half2*>(&xv);
  __half2 s = __hmul2(w[0], x[0]);
  s = __hfma2(w[1], x[1], s);
  s = __hfma2(w[2], x[2], s);
  s = __hfma2(w[3], x[3], s);
  return __low2float(s) + __high2float(s);
}

// 8-term dot product of bf16 weights with bf16 activations in f32.
__device__ __forceinline__ float dot8_bf(const uint4 w, const uint4 x) {
  float t0 = bf_lo(w.x) * bf_lo(x.x), t1 = bf_hi(w.x) * bf_hi(x.x);
  t0 = fmaf(bf_lo(w.y), bf_lo(x.y), t0); t1 = fmaf(bf_hi(w.y), bf_hi(x.y), t1);
  t0 = fmaf(bf_lo(w.z), bf_lo(x.z), t0); t1 = fmaf(bf_hi(w.z), bf_hi(x.z), t1);
  t0 = fmaf(bf_lo(w.w), bf_lo(x.w), t0); t1 = fmaf(bf_hi(w.w), bf_hi(x.w), t1);
  return t0 + t1;
}

// Group scale byte -> f32 (E8M0 for MXFP8, E4M3 for NVFP4).
template <int FMT>
__device__ __forceinline__ float scale_f(uint32_t b) {
  return FMT == WF_MXFP8 ? e8m0_f(b) : e4m3_f(b);
}

// Lane-partial dot products of R staged rows (an item each: wr[r], seg
// weights) with NB activation segments (x, row stride K elements).  Group
// scales come from the stage (sr[r], shared memory) or, when they could not
// be staged, from global memory (gr[r], already offset to the segment).
template <int FMT, int NB, int R>
__device__ __forceinline__ void item_dot(const uint8_t* const (&wr)[R],
                                         const uint8_t* const (&sr)[R],
                                         const uint8_t* const (&gr)[R],
                                         const void* x, int K, int nch,
                                         int lane, float (&acc)[R][NB]) {
  constexpr int LB = FmtInfo<FMT>::LB;
  constexpr int GSH = FMT == WF_MXFP8 ? 2 : 1;   // chunk -> group index
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;
#pragma unroll 2
  for (int c = lane; c < nch; c += 32) {
    uint4 xv[NB];
#pragma unroll
    for (int b = 0; b < NB; ++b)
      xv[b] = *reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint16_t*>(x) + (size_t)b * K + c * 8);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      if (FMT == WF_BF16) {
        const uint4 wv = *reinterpret_cast<const uint4*>(wr[r] + c * LB);
#pragma unroll
        for (int b = 0; b < NB; ++b) acc[r][b] += dot8_bf(wv, xv[b]);
      } else {
        const uint32_t sb = sr[r] ? (uint32_t)sr[r][c >> GSH]
                                  : (uint32_t)__ldg(gr[r] + (c >> GSH));
        const float sc = scale_f<FMT>(sb);
        __half2 w[4];
        decode8_h2<FMT>(wr[r] + c * LB, w);
#pragma unroll
        for (int b = 0; b < NB; ++b)
          acc[r][b] = fmaf(dot8_h2(w, xv[b]), sc, acc[r][b]);
      }
    }
  }
}

// ---- prologue: activation rows -> shared memory ---------------------------
constexpr int kU = 9;        // PRO_UPDATE: elements per thread, K <= kU * kThreads
constexpr int kCopyU = 5;    // PRO_BF16: 16-byte loads per thread in flight

template <int FMT>
__device__ __forceinline__ void put_x(void* xs, int i, float v) {
  if (FMT == WF_BF16) reinterpret_cast<bf16*>(xs)[i] = __float2bfloat16_rn(v);
  else reinterpret_cast<__half*>(xs)[i] = __float2half_rn(v);
}

// 8 bf16 -> 8 f16 (exact for the magnitudes of normalised activations).
__device__ __forceinline__ uint4 bf8_to_h8(uint4 v) {
  uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h = __floats2half2_rn(bf_lo(w[i]), bf_hi(w[i]));
    w[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// PRO_BF16: copy the caller's bf16 rows (zero rows past B), all loads of a
// thread in flight together.
template <int FMT, int NB>
__device__ __forceinline__ void stage_x_copy(const GemvArgs& a, int XS,
                                             void* xs) {
  const int vec = a.K / 8, tid = threadIdx.x;
#pragma unroll 1
  for (int b = 0; b < NB; ++b) {
    uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(xs) +
                                          (size_t)b * XS);
    const uint4* src = reinterpret_cast<const uint4*>(
        a.xin + (size_t)(b < a.B ? b : 0) * a.xin_stride);
#pragma unroll 1
    for (int i0 = tid; i0 < vec; i0 += kCopyU * kThreads) {
      uint4 v[kCopyU];
#pragma unroll
      for (int u = 0; u < kCopyU; ++u) {
        const int i = i0 + u * kThreads;
        v[u] = (b < a.B && i < vec) ? src[i] : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kCopyU; ++u) {
        const int i = i0 + u * kThreads;
        if (i < vec) dst[i] = FMT == WF_BF16 ? v[u] : bf8_to_h8(v[u]);
      }
    }
  }
}

struct UpdScal { float inv_h, inv_t, inv_u; };

// Norm reciprocals from the block-reduced sums r = [|h|^2, sum (a s)^2,
// sum (a s)(alpha h), sum (alpha h)^2, sum (a s) x, sum (alpha h) x, |x|^2],
// a = 1 - alpha.
__device__ __forceinline__ UpdScal upd_scalars(const float (&r)[7], bool next) {
  UpdScal q;
  q.inv_h = 1.f / fmaxf(sqrtf(r[0]), 1e-12f);
  const float tt = r[1] + 2.f * r[2] * q.inv_h + r[3] * q.inv_h * q.inv_h;
  q.inv_t = 1.f / fmaxf(sqrtf(fmaxf(tt, 0.f)), 1e-12f);
  q.inv_u = 1.f;
  if (next) {
    const float dot = (r[4] + r[5] * q.inv_h) * q.inv_t;
    q.inv_u = 1.f / fmaxf(sqrtf(fmaxf(1.f + 2.f * dot + r[6], 0.f)), 1e-12f);
  }
  return q;
}

// Element i of the updated row: new state (block 0 stores it, and x for
// RJ_FIRST), re-injected value to the activation row in shared memory.
template <int FMT>
__device__ __forceinline__ void upd_store(const GemvArgs& a, const UpdScal& q,
                                          int rj, size_t row, size_t xrow,
                                          int i, float al, float sv, float hv,
                                          float xv, void* xs) {
  const bool lead = blockIdx.x == 0;
  float v = ((1.f - al) * sv + al * hv * q.inv_h) * q.inv_t;
  if (rj == RJ_FIRST && lead && a.x_buf) a.x_buf[row + i] = v;
  if (rj == RJ_NEXT) v = (v + xv) * q.inv_u;
  if (lead) a.s_out[row + i] = v;
  put_x<FMT>(xs, (int)(xrow + i), v);
}

// A row sitting out this loop keeps its state (row_reinject < 0).
template <int FMT>
__device__ __forceinline__ void keep_row(const GemvArgs& a, int b, int XS,
                                         void* xs) {
  const size_t row = (size_t)b * a.K;
  for (int i = threadIdx.x; i < a.K; i += kThreads) {
    const float v = a.s_in[row + i];
    if (blockIdx.x == 0) a.s_out[row + i] = v;
    put_x<FMT>(xs, (int)((size_t)b * XS + i), v);
  }
}

// PRO_UPDATE for batch row b: the previous sublayer's nGPT update
//   s <- N((1 - alpha) s + alpha h / |h|),  h = sum of h_S partials,
// and the loop re-injection (RJ_FIRST: x := s, result s; RJ_NEXT: result
// N(s + x)), with both norms from one block reduction
//   |t|^2 = sum ((1-alpha) s)^2 + 2 sum (1-alpha) alpha s h / |h|
//           + sum (alpha h)^2 / |h|^2,
//   |t + x|^2 = 1 + 2 t.x + |x|^2   (t of unit norm).
// Every thread keeps its kU elements in registers across the reduction, so
// the whole update costs one round trip to L2.  `al` holds this thread's
// alpha values (loaded before the programmatic-dependent-launch wait).
template <int FMT>
__device__ __forceinline__ void stage_x_update(const GemvArgs& a, int b, int XS,
                                               const float (&al)[kU], void* xs,
                                               float* red) {
  const int K = a.K, tid = threadIdx.x;
  const int rj = row_reinject(a.row_loops, b, a.upd_loop, a.rj_loop, a.reinject);
  if (rj < 0) {
    keep_row<FMT>(a, b, XS, xs);
    return;
  }
  const bool next = rj == RJ_NEXT;
  const size_t row = (size_t)b * K, hs = (size_t)a.B * K;
  float sv[kU], hv[kU], xv[kU];
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int i = tid + u * kThreads;
    sv[u] = hv[u] = xv[u] = 0.f;
    if (i < K) {
      sv[u] = a.s_in[row + i];
      hv[u] = a.h_in[row + i];
      if (next) xv[u] = a.x_buf[row + i];
    }
  }
#pragma unroll 1
  for (int k0 = 1; k0 < a.h_S; k0 += 3) {
    float t[3][kU];
#pragma unroll
    for (int j = 0; j < 3; ++j)
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = tid + u * kThreads;
        t[j][u] = (k0 + j < a.h_S && i < K) ? a.h_in[(k0 + j) * hs + row + i] : 0.f;
      }
#pragma unroll
    for (int u = 0; u < kU; ++u) hv[u] += t[0][u] + t[1][u] + t[2][u];
  }
  float r[7] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const float as = (1.f - al[u]) * sv[u], ah = al[u] * hv[u];
    r[0] = fmaf(hv[u], hv[u], r[0]);
    r[1] = fmaf(as, as, r[1]);
    r[2] = fmaf(as, ah, r[2]);
    r[3] = fmaf(ah, ah, r[3]);
    r[4] = fmaf(as, xv[u], r[4]);
    r[5] = fmaf(ah, xv[u], r[5]);
    r[6] = fmaf(xv[u], xv[u], r[6]);
  }
  block_sum_n<7>(r, red);
  const UpdScal q = upd_scalars(r, next);
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int i = tid + u * kThreads;
    if (i < K)
      upd_store<FMT>(a, q, rj, row, (size_t)b * XS, i, al[u], sv[u], hv[u],
                     xv[u], xs);
  }
}

// PRO_UPDATE for K > kU * kThreads: the same update in two passes, the
// summed h kept in shared memory (tmp [K]) in between.
template <int FMT>
__device__ void stage_x_update_2pass(const GemvArgs& a, int b, int XS, void* xs,
                                     float* tmp, float* red) {
  const int K = a.K, tid = threadIdx.x;
  const int rj = row_reinject(a.row_loops, b, a.upd_loop, a.rj_loop, a.reinject);
  if (rj < 0) {
    keep_row<FMT>(a, b, XS, xs);
    return;
  }
  const bool next = rj == RJ_NEXT;
  const size_t row = (size_t)b * K, hs = (size_t)a.B * K;
  float r[7] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int i = tid; i < K; i += kThreads) {
    float h = 0.f;
    for (int k = 0; k < a.h_S; ++k) h += a.h_in[k * hs + row + i];
    const float al = a.alpha[i], sv = a.s_in[row + i];
    const float xv = next ? a.x_buf[row + i] : 0.f;
    tmp[i] = h;
    const float as = (1.f - al) * sv, ah = al * h;
    r[0] = fmaf(h, h, r[0]);
    r[1] = fmaf(as, as, r[1]);
    r[2] = fmaf(as, ah, r[2]);
    r[3] = fmaf(ah, ah, r[3]);
    r[4] = fmaf(as, xv, r[4]);
    r[5] = fmaf(ah, xv, r[5]);
    r[6] = fmaf(xv, xv, r[6]);
  }
  block_sum_n<7>(r, red);
  const UpdScal q = upd_scalars(r, next);
  for (int i = tid; i < K; i += kThreads)
    upd_store<FMT>(a, q, rj, row, (size_t)b * XS, i, a.alpha[i],
                   a.s_in[row + i], tmp[i], next ? a.x_buf[row + i] : 0.f, xs);
}

// ---- batch-1 BF16 rows on the tensor cores ---------------------------------
// One row segment w[0..seg) (seg = 256 * nks, in shared memory) dotted with
// x on the warp-level MMA: the segment is read as a 16 x (seg/16) matrix A
// whose row i holds the 8-element chunks i, i+16, i+32, ... of w, and B
// holds the matching chunks of x in its column i, so that
// sum_i (A B)[i][i] = w . x.  The off-diagonal products are discarded: the
// tensor cores have far more throughput than this needs, and in exchange x
// stays in registers (B fragments, loaded once per launch) and the weights
// are read from shared memory once, by ldmatrix (k-step s covers chunks
// 32 s .. 32 s + 31, 512 contiguous bytes).  Per row: nks ldmatrix.x4 and
// 2 nks MMAs instead of ~27 instructions per 8 weights and lane.
constexpr int kKS = kSeg / 256;           // k-steps of a full segment

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// B fragments of x segment xseg (bf16) for k-steps s < nks.  Fragment layout
// of m16n8k16 (col-major B): lane (g = lane / 4, t = lane % 4) holds k rows
// 2t, 2t+1 (reg 0) and 2t+8, 2t+9 (reg 1) of column g.  Columns 0-7 of the
// first MMA take chunks g and g+16 of k-step s, columns 8-15 of the second
// chunks g+8 and g+24.
__device__ __forceinline__ void load_xfrag(const bf16* xseg, int nks, int lane,
                                           uint32_t (&xb)[kKS][4]) {
  const int g = lane >> 2, t = lane & 3;
  const uint32_t* xw = reinterpret_cast<const uint32_t*>(xseg);
#pragma unroll
  for (int s = 0; s < kKS; ++s) {
    if (s < nks) {
      const int c0 = 32 * s + g;
      xb[s][0] = xw[(c0 + 0) * 4 + t];
      xb[s][1] = xw[(c0 + 16) * 4 + t];
      xb[s][2] = xw[(c0 + 8) * 4 + t];
      xb[s][3] = xw[(c0 + 24) * 4 + t];
    } else {
      xb[s][0] = xb[s][1] = xb[s][2] = xb[s][3] = 0u;
    }
  }
}

// Full dot product (every lane gets it) of the staged row segment at w.
__device__ __forceinline__ float row_dot_mma(const uint8_t* w,
                                             const uint32_t (&xb)[kKS][4],
                                             int nks, int lane) {
  float d[4][4] = {};                     // two accumulator pairs (ILP)
  const uint32_t base = smem_addr(w) + lane * 16;
#pragma unroll
  for (int s = 0; s < kKS; ++s) {
    if (s < nks) {
      uint32_t a[4];
      asm volatile(
          "ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
          : "=r"(a[0]), "=r"(a[1]), "=r"(a[2]), "=r"(a[3])
          : "r"(base + s * 512));
      mma_bf16_16816(d[(s & 1) * 2 + 0], a, xb[s][0], xb[s][1]);
      mma_bf16_16816(d[(s & 1) * 2 + 1], a, xb[s][2], xb[s][3]);
    }
  }
  // diagonal: (i, i) of the first MMA sits in lane 4i + i/2 (d[0] / d[1]
  // for even / odd i), (8+i, 8+i) of the second in the same lane (d[2] /
  // d[3])
  const int g = lane >> 2, t = lane & 3;
  float v = 0.f;
  if (t == (g >> 1)) {
    v = (g & 1) ? d[0][1] + d[1][3] + d[2][1] + d[3][3]
                : d[0][0] + d[1][2] + d[2][0] + d[3][2];
  }
  return warp_sum(v);
}

// ---- several BF16 activation rows on the tensor cores -----------------------
// BF16 weights with 2..8 activation rows (whole rows, or K segments taken
// segment-major so that the 8 rows of a stage share one segment):
// m16n8k16 with the activation rows as the M rows (NB of 16 used) and the 8
// weight rows of a stage as the N = 8 columns, so every product but those of
// the unused M rows counts.  Warp w takes the w-th eighth of K of all 8 rows
// (its activation fragments stay in registers for the whole launch), and the
// eight warps' partial sums meet in shared memory once per stage.
template <int NB, int EPI, int FMT>
constexpr bool kMmaB = FMT == WF_BF16 && NB >= 2 && EPI != EPI_LMHEAD;

// Row stride (elements) of the activation rows in shared memory: padded by
// 16 bytes where the batched MMA path reads them, so that the 8 rows of a
// fragment load fall in different banks.
__host__ __device__ constexpr int x_stride_of(int fmt, int nb, int K) {
  return (fmt == WF_BF16 && nb >= 2) ? K + 8 : K;
}
template <int NB, int FMT>
__device__ __forceinline__ int x_stride(int K) { return x_stride_of(FMT, NB, K); }

// Partial-sum buffer of the batched MMA path: two stages x kWarps x R x 64.
constexpr int kRedFloats = 2 * kWarps * 2 * 64;

// Barrier of the consumer warps (named barrier 1) that also ORs a flag over
// them, so that all take the same branch afterwards.
__device__ __forceinline__ bool cons_bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n"
      " bar.red.or.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(kWarps * 32)
      : "memory");
  return r != 0;
}

// ---- the kernel -----------------------------------------------------------
// Blocks per SM the kernel is compiled for: two for quantised weights, whose
// SIMT decode loop is bound by the latency of its dependent chains (twice
// the warps hide it: MXFP8 batch-1 decode 267 -> 328 tok/s, NVFP4
// 285 -> 355, k = 2); one for BF16, whose batch-1 rows run on the warp MMA
// and whose batched SIMT rows measured slower with two blocks (batch 4 at a
// 131K context 461 -> 436 tok/s).
template <int NB, int FMT>
constexpr int kBlocksPerSm = FMT != WF_BF16 ? 2 : 1;

template <int NB, int EPI, int FMT>
__global__ void __launch_bounds__(kThreads, (kBlocksPerSm<NB, FMT>))
gemv_kernel(const GemvArgs a, const Plan pl) {
  constexpr int R = (EPI == EPI_SWIGLU) ? 2 : 1;
  constexpr int LB = FmtInfo<FMT>::LB;       // bytes per 8 weights
  constexpr int GROUP = FMT == WF_MXFP8 ? 32 : 16;
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = a.K, S = pl.S, NS = pl.NS;
  const int seg = K >> pl.sh, nch = seg / 8;
  const uint32_t item_bytes = (uint32_t)nch * LB;
  // quantised formats: each item's group scales (sb bytes) ride in the same
  // stage as its codes when they keep the 16-byte rules of bulk copies,
  // else the consumers read them from global memory
  const int sb = FMT == WF_BF16 ? 0 : seg / GROUP;
  const bool sc_tma = FMT != WF_BF16 && (sb % 16) == 0;
  // several BF16 activation rows with whole-row items: the 8 rows of a
  // stage are the 8 MMA columns (see mma_rows8), each item copied to its own
  // 16-byte-padded slot so that ldmatrix reads them without bank conflicts
  // (K-split items only from 4 rows on: with 2 rows the per-segment
  // fragment reloads cost more than the SIMT loop, 531 -> 495 tok/s)
  const bool mmab = kMmaB<NB, EPI, FMT> && a.n_items % 8 == 0 &&
                    (S == 1 || NB >= 4);
  const uint32_t item_pitch = item_bytes + (mmab ? 16u : 0u);
  const uint32_t codes_bytes = (uint32_t)kWarps * R * item_pitch;
  const uint32_t stage_bytes =
      codes_bytes + (sc_tma ? (uint32_t)(kWarps * R * sb) : 0u);
  const int XS = x_stride<NB, FMT>(K);                    // activation row
  uint8_t* ring = smem;                                   // NS stages
  void* xs = ring + (size_t)NS * stage_bytes;             // [NB][XS] 16-bit
  float* tmp = reinterpret_cast<float*>(reinterpret_cast<uint16_t*>(xs) +
                                        (size_t)NB * XS); // [K] if 2-pass
  uint64_t* full = reinterpret_cast<uint64_t*>(tmp + (pl.tmp ? K : 0));
  uint64_t* empty = full + NS;
  __shared__ float red[7 * (kWarps + 1)];
  __shared__ float bestv[kWarps][NB];
  __shared__ int besti[kWarps][NB];
  __shared__ int s_fail, s_issued;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // item range.  Row-major items (row it >> sh, segment it & (S - 1)): a
  // stage of 8 items starts at a multiple of S, so warp w always works on K
  // segment w % S.  Batched MMA path with S > 1: segment-major items
  // (segment it / n_items, row it % n_items) in ranges aligned to 8, so the
  // 8 rows of a stage share one K segment.
  int j0 = (int)((long)a.n_items * blockIdx.x / gridDim.x) * S;
  int j1 = (int)((long)a.n_items * (blockIdx.x + 1) / gridDim.x) * S;
  if (mmab && S > 1) {
    const long tot = (long)a.n_items * S;
    j0 = (int)(tot * blockIdx.x / gridDim.x) & ~7;
    j1 = blockIdx.x + 1 == gridDim.x ? (int)tot
                                     : (int)(tot * (blockIdx.x + 1) / gridDim.x) & ~7;
  }
  const int n_stages = (j1 - j0 + kWarps - 1) / kWarps;
  const bool producer = tid == kWarps * 32;

  // items j0.. are contiguous in W: item it = (row it >> sh, segment it & (S-1))
  const uint64_t pol = evict_first_policy();
  auto issue = [&](int s) {
    const int it = j0 + s * kWarps;
    const int cnt = j1 - it < kWarps ? j1 - it : kWarps;
    const uint32_t bytes = (uint32_t)cnt * item_bytes;
    uint64_t* bar = full + (s % NS);
    uint8_t* dst = ring + (size_t)(s % NS) * stage_bytes;
    const char* w = FMT == WF_BF16 ? reinterpret_cast<const char*>(a.W)
                                   : reinterpret_cast<const char*>(a.Wq);
    const uint32_t sbytes = sc_tma ? (uint32_t)(cnt * sb) : 0u;
    mbar_expect_tx(bar, (bytes + sbytes) * R);
    if (mmab) {
      for (int k = 0; k < cnt; ++k) {
        // segment-major item it + k: row (it + k) % n_items, segment (it + k) / n_items
        const size_t src = (size_t)((it + k) % a.n_items) * S + (it + k) / a.n_items;
        tma_load_1d_hint(dst + k * item_pitch, w + src * item_bytes, item_bytes,
                         bar, pol);
        if (R == 2)
          tma_load_1d_hint(dst + (kWarps + k) * item_pitch,
                           w + ((size_t)it + k + (size_t)a.pair_off) * item_bytes,
                           item_bytes, bar, pol);
      }
    } else {
      tma_load_1d_hint(dst, w + (size_t)it * item_bytes, bytes, bar, pol);
      if (R == 2)
        tma_load_1d_hint(dst + kWarps * item_bytes,
                         w + ((size_t)it + (size_t)a.pair_off * S) * item_bytes,
                         bytes, bar, pol);
    }
    if (sc_tma) {
      // scales of item it start at byte it * sb (rows are K / GROUP bytes)
      const char* ws = reinterpret_cast<const char*>(a.Ws);
      tma_load_1d_hint(dst + codes_bytes, ws + (size_t)it * sb, sbytes, bar, pol);
      if (R == 2)
        tma_load_1d_hint(dst + codes_bytes + kWarps * sb,
                         ws + ((size_t)it + (size_t)a.pair_off * S) * sb, sbytes,
                         bar, pol);
    }
  };

  // alpha is a weight: read it before the wait, like the first stages
  float al[kU];
  const bool upd_reg = a.pro == PRO_UPDATE && !pl.tmp;
#pragma unroll
  for (int u = 0; u < kU; ++u) {
    const int i = tid + u * kThreads;
    al[u] = (upd_reg && i < K) ? __ldg(a.alpha + i) : 0.f;
  }
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
  if (a.pro == PRO_UPDATE) {
#pragma unroll 1
    for (int b = 0; b < NB; ++b) {
      if (b < a.B) {
        if (upd_reg) stage_x_update<FMT>(a, b, XS, al, xs, red);
        else stage_x_update_2pass<FMT>(a, b, XS, xs, tmp, red);
      } else {
        for (int i = tid; i < K; i += kThreads) put_x<FMT>(xs, b * XS + i, 0.f);
      }
    }
  } else {
    stage_x_copy<FMT, NB>(a, XS, xs);
  }
  __syncthreads();

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
    // ---- consumers -----------------------------------------------------
    const int sbrow = FMT == WF_BF16 ? 0 : K / GROUP;
    int slot = 0;
    uint32_t phase = 0;
    bool done = false;
    if constexpr (kMmaB<NB, EPI, FMT>) {
      if (mmab) {
        done = true;
        constexpr int KSW = kSeg / (16 * kWarps);   // k-steps per warp, max
        const int ksw = seg / (16 * kWarps);        // even: seg % 256 == 0
        const int kb = warp * ksw * 16;             // this warp's first k
        const int g = lane >> 2, t = lane & 3, ct = tid;
        uint32_t af[KSW][2];
        const uint16_t* xh = reinterpret_cast<const uint16_t*>(xs);
        // activation fragments of K segment sg (kept while the segment lasts)
        int aseg = -1;
        auto load_af = [&](int sg) {
#pragma unroll
          for (int q = 0; q < KSW; ++q) {
            af[q][0] = af[q][1] = 0u;
            if (q < ksw && g < NB) {
              const uint16_t* xr =
                  xh + (size_t)g * XS + (size_t)sg * seg + kb + 16 * q + 2 * t;
              af[q][0] = *reinterpret_cast<const uint32_t*>(xr);
              af[q][1] = *reinterpret_cast<const uint32_t*>(xr + 8);
            }
          }
          aseg = sg;
        };
        float* redm = reinterpret_cast<float*>(full + 2 * kMaxStages);
        // ldmatrix.x4 of two k-steps: lane l addresses row l % 8 of matrix
        // l / 8 (k offsets 0, 8, 16, 24)
        const uint32_t loff = (uint32_t)(lane & 7) * item_pitch +
                              (uint32_t)(kb + 8 * (lane >> 3)) * 2;
        for (int s = 0; s < n_stages; ++s) {
          const int it0 = j0 + s * kWarps;
          const int cnt = j1 - it0 < kWarps ? j1 - it0 : kWarps;
          const int sg = it0 / a.n_items, row0 = it0 - sg * a.n_items;
          if (sg != aseg) load_af(sg);
          const bool got = mbar_wait(full + slot, phase);
          if (!got && lane == 0) atomicOr(&s_fail, 1);
          float d[R][4];
#pragma unroll
          for (int r = 0; r < R; ++r) d[r][0] = d[r][1] = d[r][2] = d[r][3] = 0.f;
          if (got) {
            const uint32_t sbase = smem_addr(ring + (size_t)slot * stage_bytes);
#pragma unroll
            for (int r = 0; r < R; ++r) {
              const uint32_t rb = sbase + (uint32_t)(r * kWarps) * item_pitch + loff;
#pragma unroll
              for (int q = 0; q < KSW; q += 2) {
                if (q < ksw) {
                  uint32_t b[4];
                  asm volatile(
                      "ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                      : "=r"(b[0]), "=r"(b[1]), "=r"(b[2]), "=r"(b[3])
                      : "r"(rb + q * 32));
                  const uint32_t a0[4] = {af[q][0], 0u, af[q][1], 0u};
                  const uint32_t a1[4] = {af[q + 1][0], 0u, af[q + 1][1], 0u};
                  mma_bf16_16816(d[r], a0, b[0], b[1]);
                  mma_bf16_16816(d[r], a1, b[2], b[3]);
                }
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty + slot);   // stage read
          }
          // partial sums: lane (g, t) holds D[g][2t], D[g][2t + 1] (batch
          // row g, weight rows 2t, 2t + 1 of the stage)
          float* rbuf = redm + ((size_t)(s & 1) * kWarps + warp) * R * 64;
          if (g < NB) {
#pragma unroll
            for (int r = 0; r < R; ++r) {
              rbuf[r * 64 + g * 8 + 2 * t] = d[r][0];
              rbuf[r * 64 + g * 8 + 2 * t + 1] = d[r][1];
            }
          }
          if (cons_bar_or(*fail != 0)) break;
          if (ct < NB * 8) {
            const int bb = ct >> 3, n8 = ct & 7;
            if (n8 < cnt && bb < a.B) {
              float acc[R];
#pragma unroll
              for (int r = 0; r < R; ++r) {
                acc[r] = 0.f;
#pragma unroll
                for (int w2 = 0; w2 < kWarps; ++w2)
                  acc[r] += redm[((size_t)(s & 1) * kWarps + w2) * R * 64 +
                                 r * 64 + bb * 8 + n8];
              }
              const int n = row0 + n8;
              if (EPI == EPI_F32) {
                a.out[((size_t)sg * a.B + bb) * a.n_items + n] = acc[0];
              } else {
                const float gv = acc[0];
                a.out_bf[(size_t)bb * a.pair_off + n] =
                    __float2bfloat16_rn(gv * sigmoidf_(gv) * acc[R - 1]);
              }
            }
          }
          if (++slot == NS) { slot = 0; phase ^= 1u; }
        }
      }
    }
    if (!done) {
    // ---- warp w owns item w of every stage ---------------------------------
    // batch 1, BF16: tensor-core row dots with x (this warp's segment
    // w % S) held as MMA fragments for the whole launch
    constexpr bool kMma = FMT == WF_BF16 && NB == 1;
    uint32_t xb[kMma ? kKS : 1][4];
    if constexpr (kMma)
      load_xfrag(reinterpret_cast<const bf16*>(xs) + (warp % S) * seg, seg / 256,
                 lane, reinterpret_cast<uint32_t (&)[kKS][4]>(xb));
    for (int s = 0; s < n_stages; ++s) {
      const int it = j0 + s * kWarps + warp;
      const bool has = it < j1;
      const int n = it >> pl.sh, sidx = it & (S - 1);
      if (!mbar_wait(full + slot, phase)) {
        if (lane == 0) atomicOr(&s_fail, 1);
        break;
      }
      if (has) {
        const uint8_t* stg = ring + (size_t)slot * stage_bytes;
        const uint8_t* wr[R];
        const uint8_t* sr[R];
        const uint8_t* gr[R];
#pragma unroll
        for (int r = 0; r < R; ++r) {
          wr[r] = stg + (r * kWarps + warp) * item_bytes;
          sr[r] = sc_tma ? stg + codes_bytes + (r * kWarps + warp) * sb : nullptr;
          gr[r] = (FMT != WF_BF16 && !sc_tma)
                      ? a.Ws + (size_t)(n + r * a.pair_off) * sbrow + sidx * sb
                      : nullptr;
        }
        float acc[R][NB];
        if constexpr (kMma) {
#pragma unroll
          for (int r = 0; r < R; ++r)
            acc[r][0] = row_dot_mma(wr[r], reinterpret_cast<const uint32_t (&)[kKS][4]>(xb),
                                    seg / 256, lane);
        } else {
          item_dot<FMT, NB, R>(wr, sr, gr,
                               reinterpret_cast<const uint16_t*>(xs) + sidx * seg,
                               XS, nch, lane, acc);
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[r][b] = warp_sum(acc[r][b]);
        }
        if (FMT == WF_NVFP4) {            // per-tensor second-level scale
          const float ts = __ldg(a.Wt);
#pragma unroll
          for (int r = 0; r < R; ++r)
#pragma unroll
            for (int b = 0; b < NB; ++b) acc[r][b] *= ts;
        }
        if (lane == 0) {
          const float scl = EPI == EPI_LMHEAD ? a.col_scale[n] : 0.f;
#pragma unroll
          for (int b = 0; b < NB; ++b) {
            if (b >= a.B) break;
            if (EPI == EPI_F32) {
              a.out[((size_t)sidx * a.B + b) * a.n_items + n] = acc[0][b];
            } else if (EPI == EPI_SWIGLU) {
              const float g = acc[0][b];
              a.out_bf[(size_t)b * a.pair_off + n] =
                  __float2bfloat16_rn(g * sigmoidf_(g) * acc[R - 1][b]);
            } else {
              const float z = scl * acc[0][b];
              if (a.out) a.out[(size_t)b * a.out_stride + n] = z;
              if (z > bv[b]) { bv[b] = z; bi[b] = n; }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + slot);
      if (++slot == NS) { slot = 0; phase ^= 1u; }
      if (*fail) break;
    }
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

bool needs_tmp(const GemvArgs& a) {
  return a.pro == PRO_UPDATE && a.K > kU * kThreads;
}

// Bytes of one lane chunk (8 weights) of a format.
int lane_bytes(int fmt) { return fmt == WF_BF16 ? 16 : fmt == WF_MXFP8 ? 8 : 4; }

// Host view of the batched MMA path (kMmaB and 8 | n_items).
bool mmab_kernel(const GemvArgs& a, int nb) {
  return a.fmt == WF_BF16 && nb >= 2 && a.epi != EPI_LMHEAD &&
         a.n_items % 8 == 0;
}

size_t fixed_smem(const GemvArgs& a, int nb) {
  return (size_t)nb * x_stride_of(a.fmt, nb, a.K) * 2 +
         (needs_tmp(a) ? (size_t)a.K * 4 : 0) + 2 * kMaxStages * 8 +
         (mmab_kernel(a, nb) ? (size_t)kRedFloats * 4 : 0);
}

// Bytes of one item slot in a stage (padded on the batched MMA path).
size_t item_slot(const GemvArgs& a, int nb, int S) {
  return (size_t)(a.K / S) / 8 * lane_bytes(a.fmt) +
         (mmab_kernel(a, nb) && (S == 1 || nb >= 4) ? 16 : 0);
}


// Segments per row S (F32 only: SwiGLU and LM head need whole rows) and
// ring depth: the largest segment <= kSeg whose 8-item stages still fit at
// least 3 deep (2 as a last resort).
// Blocks per SM wanted for these arguments (kBlocksPerSm of the variant the
// launcher picks; DORY_GEMV_BPS = 1 or 2 overrides it for measurements).
int bps_wanted(const GemvArgs& a, int nb) {
  (void)nb;
  const char* e = getenv("DORY_GEMV_BPS");
  if (e && atoi(e) < 2) return 1;
  return a.fmt != WF_BF16 ? 2 : 1;
}

Plan make_plan(const GemvArgs& a, int nb) {
  const int R = a.epi == EPI_SWIGLU ? 2 : 1;
  const size_t fixed = fixed_smem(a, nb);
  const int lb = lane_bytes(a.fmt);
  int bps = bps_wanted(a, nb);
  // two blocks share the SM's shared memory (and its 1 KB per block)
  size_t budget = bps == 2 ? kSmemBudget / 2 - 2048 : kSmemBudget;
  int S = 1;
  if (a.epi == EPI_F32) {
    while (a.K / S > kSeg && (a.K / (2 * S)) % 256 == 0) S *= 2;
    while ((a.K / (2 * S)) % 256 == 0 &&
           fixed + 3 * (size_t)kWarps * R * (a.K / S) / 8 * lb > budget)
      S *= 2;
  }
  const int sbytes = a.fmt == WF_BF16 ? 0
                     : (a.K / S) / (a.fmt == WF_MXFP8 ? 32 : 16);
  const size_t stage = (size_t)kWarps * R * (item_slot(a, nb, S) +
                                             (sbytes % 16 == 0 ? sbytes : 0));
  int NS = stages_default();
  if (a.fmt != WF_BF16) NS = kMaxStages;          // smaller items: go deeper
  if (bps == 2 && fixed + 2 * stage > budget) {   // two rings do not fit
    bps = 1;
    budget = kSmemBudget;
  }
  while (NS > 2 && fixed + NS * stage > budget) --NS;
  int sh = 0;
  while ((1 << sh) < S) ++sh;
  return Plan{S, sh, NS, needs_tmp(a) ? 1 : 0, bps};
}

size_t smem_bytes(const GemvArgs& a, const Plan& p, int nb) {
  const int R = a.epi == EPI_SWIGLU ? 2 : 1;
  const int sbytes = a.fmt == WF_BF16 ? 0
                     : (a.K / p.S) / (a.fmt == WF_MXFP8 ? 32 : 16);
  return (size_t)p.NS * kWarps * R *
             (item_slot(a, nb, p.S) + (sbytes % 16 == 0 ? sbytes : 0)) +
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

// The same decode for a whole matrix, written as bf16 (the products have at
// most 8 significant bits: exact); one thread per 8 consecutive weights,
// 16-byte stores.
template <int FMT>
__global__ void dequant_bf16_kernel(const uint8_t* Wq, const uint8_t* Ws,
                                    long N, int K, bf16* out) {
  pdl_wait();
  pdl_trigger();
  const long total = N * (K / 8);
  for (long id = blockIdx.x * (long)blockDim.x + threadIdx.x; id < total;
       id += (long)gridDim.x * blockDim.x) {
    const long row = id / (K / 8);
    const int k = (int)(id - row * (K / 8)) * 8;
    float w[8];
    decode8<FMT>(Wq + (row * K + k) / 8 * FmtInfo<FMT>::LB, w);
    const float sc = group_scale<FMT>(Ws, K, row, k);
    uint4 u;
    uint32_t* q = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h =
          __floats2bfloat162_rn(w[2 * e] * sc, w[2 * e + 1] * sc);
      q[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(out + row * K + k) = u;
  }
}

}  // namespace

void launch_dequant_bf16(int fmt, const uint8_t* Wq, const uint8_t* Ws, long N,
                         int K, bf16* out, cudaStream_t st) {
  const dim3 grid(148 * 8), block(256);
  if (fmt == WF_MXFP8)
    launch_k(dequant_bf16_kernel<WF_MXFP8>, grid, block, 0, st, Wq, Ws, N, K,
             out);
  else
    launch_k(dequant_bf16_kernel<WF_NVFP4>, grid, block, 0, st, Wq, Ws, N, K,
             out);
}

int gemv_splits(const GemvArgs& a) { return make_plan(a, nb_of(a.B)).S; }

int gemv_grid(const GemvArgs& a, int num_sms) {
  const int n = num_sms * make_plan(a, nb_of(a.B)).bps;
  return a.n_items < n ? a.n_items : n;
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
