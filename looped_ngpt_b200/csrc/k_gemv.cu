// Weight-streaming GEMV for small-batch decode (B <= 8 rows of activations).
//
// y[b][n] = sum_k W[n][k] x[b][k] with W bf16 row-major streamed once from
// HBM (16-byte L1-bypassing loads, several rows' loads in flight per lane)
// and x staged in shared memory as bf16.  One warp owns one work item (an
// output row, or a (row, K-segment) pair when split-K is used), so no
// cross-warp reduction is needed; split-K partials are summed by the
// consumer.
//
// Prologue PRO_UPDATE fuses the previous sublayer's nGPT residual update
// (s <- N(s + alpha (N(h) - s)), "Dory1.0-4B: A Looped Normalized-GPT" §2)
// and the loop-boundary re-injection u_t = N(s_{t-1} + x) (paper summary,
// 核心方法) into this GEMV: every block recomputes the d-length update from
// L2-resident vectors and block 0 writes the new state, so no separate
// launch or grid-wide synchronisation is needed.
//
// Epilogues: EPI_F32 (plain), EPI_SWIGLU (rows n and n + F of the fused
// gate/up matrix -> silu(gate) * up as bf16; the L2 norm that precedes the
// down projection is dropped because the normalised update makes it a
// no-op: N(W N(m)) = N(W m)), EPI_LMHEAD (logit scale s_z, optional logits
// store, per-block greedy argmax partials).
#include "common.cuh"

namespace dory {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kUnroll = 4;

template <int NB, int R>
__device__ __forceinline__ void fma_chunk(float (&acc)[R][NB],
                                          const uint4 (&w)[R],
                                          const bf16* xs, int K, int k) {
#pragma unroll
  for (int b = 0; b < NB; ++b) {
    const uint4 xv = *reinterpret_cast<const uint4*>(xs + b * K + k);
    const float x0 = bf_lo(xv.x), x1 = bf_hi(xv.x), x2 = bf_lo(xv.y),
                x3 = bf_hi(xv.y), x4 = bf_lo(xv.z), x5 = bf_hi(xv.z),
                x6 = bf_lo(xv.w), x7 = bf_hi(xv.w);
#pragma unroll
    for (int r = 0; r < R; ++r) {
      float a = acc[r][b];
      a = fmaf(bf_lo(w[r].x), x0, a);
      a = fmaf(bf_hi(w[r].x), x1, a);
      a = fmaf(bf_lo(w[r].y), x2, a);
      a = fmaf(bf_hi(w[r].y), x3, a);
      a = fmaf(bf_lo(w[r].z), x4, a);
      a = fmaf(bf_hi(w[r].z), x5, a);
      a = fmaf(bf_lo(w[r].w), x6, a);
      a = fmaf(bf_hi(w[r].w), x7, a);
      acc[r][b] = a;
    }
  }
}

template <int NB, int EPI>
__global__ void __launch_bounds__(kThreads)
gemv_kernel(const GemvArgs a) {
  constexpr int R = (EPI == EPI_SWIGLU) ? 2 : 1;
  extern __shared__ uint4 smem_raw[];
  bf16* xs = reinterpret_cast<bf16*>(smem_raw);          // [NB][K]
  float* tmp = reinterpret_cast<float*>(xs + NB * a.K);  // [K]
  __shared__ float red[kWarps];
  __shared__ float bestv[kWarps][NB];
  __shared__ int besti[kWarps][NB];
  const int K = a.K;

  // ---- prologue: activation vector(s) -> shared memory (bf16) ----------
  if (a.pro == PRO_BF16) {
    const int vec = K / 8;
    for (int b = 0; b < NB; ++b) {
      uint4* dst = reinterpret_cast<uint4*>(xs + b * K);
      if (b < a.B) {
        const uint4* src =
            reinterpret_cast<const uint4*>(a.xin + (size_t)b * a.xin_stride);
        for (int i = threadIdx.x; i < vec; i += kThreads) dst[i] = src[i];
      } else {
        for (int i = threadIdx.x; i < vec; i += kThreads)
          dst[i] = make_uint4(0, 0, 0, 0);
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
        for (int i = threadIdx.x; i < K; i += kThreads)
          xs[b * K + i] = __float2bfloat16_rn(0.f);
      }
    }
  }
  __syncthreads();

  // ---- main loop: one warp per work item --------------------------------
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int S = (EPI == EPI_F32) ? a.S : 1;
  const int seg = K / S;
  const int total = a.n_items * S;
  float bv[NB];
  int bi[NB];
#pragma unroll
  for (int b = 0; b < NB; ++b) { bv[b] = -INFINITY; bi[b] = 0x7fffffff; }

  for (int it = blockIdx.x * kWarps + warp; it < total;
       it += gridDim.x * kWarps) {
    const int n = it / S, sidx = it - n * S;
    const int k0 = sidx * seg;
    const bf16* wr[R];
    wr[0] = a.W + (size_t)n * K + k0;
    if (R == 2) wr[R - 1] = a.W + (size_t)(n + a.pair_off) * K + k0;
    float acc[R][NB];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[r][b] = 0.f;

    int k = lane * 8;
    for (; k + 256 * (kUnroll - 1) < seg; k += 256 * kUnroll) {
      uint4 w[kUnroll][R];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
#pragma unroll
        for (int r = 0; r < R; ++r) w[u][r] = ld_stream(wr[r] + k + u * 256);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        fma_chunk<NB, R>(acc, w[u], xs, K, k0 + k + u * 256);
    }
    for (; k < seg; k += 256) {
      uint4 w[R];
#pragma unroll
      for (int r = 0; r < R; ++r) w[r] = ld_stream(wr[r] + k);
      fma_chunk<NB, R>(acc, w, xs, K, k0 + k);
    }
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < NB; ++b) acc[r][b] = warp_sum(acc[r][b]);

    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < NB; ++b) {
        if (b >= a.B) break;
        if (EPI == EPI_F32) {
          a.out[((size_t)sidx * a.B + b) * a.n_items + n] = acc[0][b];
        } else if (EPI == EPI_SWIGLU) {
          const float g = acc[0][b];
          const float m = g * sigmoidf_(g) * acc[R - 1][b];
          a.out_bf[(size_t)b * a.pair_off + n] = __float2bfloat16_rn(m);
        } else {
          const float z = a.col_scale[n] * acc[0][b];
          if (a.out) a.out[(size_t)b * a.out_stride + n] = z;
          if (z > bv[b]) { bv[b] = z; bi[b] = n; }
        }
      }
    }
  }

  if (EPI == EPI_LMHEAD) {
    if (lane == 0) {
#pragma unroll
      for (int b = 0; b < NB; ++b) { bestv[warp][b] = bv[b]; besti[warp][b] = bi[b]; }
    }
    __syncthreads();
    if (threadIdx.x < a.B && threadIdx.x < NB) {
      const int b = threadIdx.x;
      float v = -INFINITY;
      int idx = 0x7fffffff;
      for (int w = 0; w < kWarps; ++w) {
        const float c = bestv[w][b];
        const int ci = besti[w][b];
        if (c > v || (c == v && ci < idx)) { v = c; idx = ci; }
      }
      a.amax_val[b * gridDim.x + blockIdx.x] = v;
      a.amax_idx[b * gridDim.x + blockIdx.x] = idx;
    }
  }
}

template <int NB, int EPI>
void launch_t(const GemvArgs& a, int grid, cudaStream_t st) {
  const size_t smem = (size_t)NB * a.K * sizeof(bf16) +
                      (a.pro == PRO_UPDATE ? (size_t)a.K * sizeof(float) : 0);
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    cudaFuncSetAttribute(gemv_kernel<NB, EPI>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    configured = smem;
  }
  gemv_kernel<NB, EPI><<<grid, kThreads, smem, st>>>(a);
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

int gemv_grid(const GemvArgs& a, int num_sms) {
  const int S = (a.epi == EPI_F32) ? a.S : 1;
  const long total = (long)a.n_items * S;
  const long want = (total + kWarps - 1) / kWarps;
  const int nb = a.B <= 1 ? 1 : a.B <= 2 ? 2 : a.B <= 4 ? 4 : 8;
  const size_t smem = (size_t)nb * a.K * 2 + (a.pro == PRO_UPDATE ? a.K * 4 : 0);
  int per_sm = (int)((200 * 1024) / (smem + 1024));
  if (per_sm > 4) per_sm = 4;
  if (per_sm < 1) per_sm = 1;
  const long cap = (long)num_sms * per_sm;
  return (int)(want < cap ? want : cap);
}

void launch_gemv(const GemvArgs& a, int grid, cudaStream_t st) {
  if (a.B <= 1) launch_nb<1>(a, grid, st);
  else if (a.B <= 2) launch_nb<2>(a, grid, st);
  else if (a.B <= 4) launch_nb<4>(a, grid, st);
  else launch_nb<8>(a, grid, st);
}

}  // namespace dory
