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

// Dot products of one staged row segment (kl elements) with the NB
// activation rows; returns the warp-reduced sums in every lane.
template <int NB>
__device__ __forceinline__ void row_slice_dot(const bf16* wrow, const bf16* xk,
                                              int K, int kl, int lane,
                                              float (&acc)[NB]) {
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = 0.f;
#pragma unroll 5
  for (int k = lane * 8; k < kl; k += 256) {
    const uint4 wv = *reinterpret_cast<const uint4*>(wrow + k);
    const float w0 = bf_lo(wv.x), w1 = bf_hi(wv.x), w2 = bf_lo(wv.y),
                w3 = bf_hi(wv.y), w4 = bf_lo(wv.z), w5 = bf_hi(wv.z),
                w6 = bf_lo(wv.w), w7 = bf_hi(wv.w);
#pragma unroll
    for (int b = 0; b < NB; ++b) {
      const uint4 xv = *reinterpret_cast<const uint4*>(xk + b * K + k);
      float t = acc[b];
      t = fmaf(w0, bf_lo(xv.x), t);
      t = fmaf(w1, bf_hi(xv.x), t);
      t = fmaf(w2, bf_lo(xv.y), t);
      t = fmaf(w3, bf_hi(xv.y), t);
      t = fmaf(w4, bf_lo(xv.z), t);
      t = fmaf(w5, bf_hi(xv.z), t);
      t = fmaf(w6, bf_lo(xv.w), t);
      t = fmaf(w7, bf_hi(xv.w), t);
      acc[b] = t;
    }
  }
#pragma unroll
  for (int b = 0; b < NB; ++b) acc[b] = warp_sum(acc[b]);
}

// One staged row segment times the register-resident x slice (batch 1):
// lane covers elements c * 256 + lane * 8 + [0, 8) for c < nc.  Two
// accumulators break the FMA dependency chain.
template <int MAXC>
__device__ __forceinline__ float row_dot_reg(const bf16* wrow, const float* xr,
                                             int nc, int lane) {
  float a0 = 0.f, a1 = 0.f;
  const bf16* wp = wrow + lane * 8;
#pragma unroll
  for (int c = 0; c < MAXC; ++c) {
    if (c < nc) {
      const uint4 wv = *reinterpret_cast<const uint4*>(wp + c * 256);
      a0 = fmaf(bf_lo(wv.x), xr[c * 8 + 0], a0);
      a1 = fmaf(bf_hi(wv.x), xr[c * 8 + 1], a1);
      a0 = fmaf(bf_lo(wv.y), xr[c * 8 + 2], a0);
      a1 = fmaf(bf_hi(wv.y), xr[c * 8 + 3], a1);
      a0 = fmaf(bf_lo(wv.z), xr[c * 8 + 4], a0);
      a1 = fmaf(bf_hi(wv.z), xr[c * 8 + 5], a1);
      a0 = fmaf(bf_lo(wv.w), xr[c * 8 + 6], a0);
      a1 = fmaf(bf_hi(wv.w), xr[c * 8 + 7], a1);
    }
  }
  return warp_sum(a0 + a1);
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


template <int NB, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
gemv_kernel(const GemvArgs a, const Plan pl) {
  constexpr int R = (EPI == EPI_SWIGLU) ? 2 : 1;
  extern __shared__ __align__(128) uint8_t smem[];
  const int K = a.K, S = pl.S, NS = pl.NS;
  const int seg = K / S;
  const size_t item_bytes = (size_t)seg * sizeof(bf16);
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
    const char* w = reinterpret_cast<const char*>(a.W);
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
      if (!mbar_wait(full + slot, (uint32_t)((s / NS) & 1))) {
        if (lane == 0) atomicOr(&s_fail, 1);
        break;
      }
      const long it = j0 + (long)s * kWarps + warp;
      if (it < j1) {
        const int n = (int)(it / S), sidx = (int)(it - (long)n * S);
        float scl = 0.f;
        if (EPI == EPI_LMHEAD && lane == 0) scl = a.col_scale[n];
        const bf16* wrow = reinterpret_cast<const bf16*>(
            ring + slot * stage_bytes + warp * item_bytes);
        float acc[NB], acc2[NB];
        if (NB == 1) {
          acc[0] = row_dot_reg<kMaxC>(wrow, xr, nc, lane);
          if (R == 2) acc2[0] = row_dot_reg<kMaxC>(wrow + kWarps * seg, xr, nc, lane);
        } else {
          row_slice_dot<NB>(wrow, xs + sidx * seg, K, seg, lane, acc);
          if (R == 2)
            row_slice_dot<NB>(wrow + kWarps * seg, xs, K, seg, lane, acc2);
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
Plan make_plan(const GemvArgs& a, int nb) {
  const int R = a.epi == EPI_SWIGLU ? 2 : 1;
  const size_t fixed = fixed_smem(a, nb);
  int S = 1;
  if (a.epi == EPI_F32) {
    while (a.K / S > kSeg && (a.K / (2 * S)) % 256 == 0) S *= 2;
    while ((a.K / (2 * S)) % 256 == 0 &&
           fixed + 3 * (size_t)kWarps * R * (a.K / S) * 2 > kSmemBudget)
      S *= 2;
  }
  const size_t stage = (size_t)kWarps * R * (a.K / S) * 2;
  int NS = stages_default();
  while (NS > 2 && fixed + NS * stage > kSmemBudget) --NS;
  return Plan{S, NS};
}

size_t smem_bytes(const GemvArgs& a, const Plan& p, int nb) {
  const int R = a.epi == EPI_SWIGLU ? 2 : 1;
  return (size_t)p.NS * kWarps * R * (a.K / p.S) * 2 + fixed_smem(a, nb);
}

int nb_of(int B) { return B <= 1 ? 1 : B <= 2 ? 2 : B <= 4 ? 4 : 8; }

template <int NB, int EPI>
void launch_t(const GemvArgs& a, int grid, cudaStream_t st) {
  const Plan pl = make_plan(a, NB);
  const size_t smem = smem_bytes(a, pl, NB);
  static size_t configured = 0;
  if (smem > configured) {
    cudaFuncSetAttribute(gemv_kernel<NB, EPI>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    configured = smem;
  }
  launch_k(gemv_kernel<NB, EPI>, dim3(grid), dim3(kThreads), smem, st, a, pl);
}

template <int NB>
void launch_nb(const GemvArgs& a, int grid, cudaStream_t st) {
  switch (a.epi) {
    case EPI_F32: launch_t<NB, EPI_F32>(a, grid, st); break;
    case EPI_SWIGLU: launch_t<NB, EPI_SWIGLU>(a, grid, st); break;
    default: launch_t<NB, EPI_LMHEAD>(a, grid, st); break;
  }
}

}  // namespace

int gemv_splits(const GemvArgs& a) { return make_plan(a, nb_of(a.B)).S; }

int gemv_grid(const GemvArgs& a, int num_sms) {
  return a.n_items < num_sms ? a.n_items : num_sms;
}

void launch_gemv(const GemvArgs& a, int grid, cudaStream_t st) {
  if (a.B <= 1) launch_nb<1>(a, grid, st);
  else if (a.B <= 2) launch_nb<2>(a, grid, st);
  else if (a.B <= 4) launch_nb<4>(a, grid, st);
  else launch_nb<8>(a, grid, st);
}

}  // namespace dory
