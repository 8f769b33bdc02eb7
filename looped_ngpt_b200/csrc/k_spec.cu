// Acceptance step of self-speculative decoding ("Dory1.0-4B: A Looped
// Normalized-GPT", §6.2 Self-Speculative Decoding: the k = 1 model drafts
// gamma tokens, the k = 4 model verifies them in one pass, rejection
// sampling keeps the output distribution of the verifier).
//
// The draft is greedy (each draft token is the k = 1 model's argmax, a point
// mass q = delta(d)).  For such a draft the rejection-sampling rule of
// speculative sampling reads: draft token d_j is accepted with probability
// p(d_j), p the verifier's distribution at that position; at the first
// rejection the token is drawn from p restricted to x != d_j (the residual
// max(0, p - q), renormalised); if every draft is accepted, one more token
// is drawn from p at the last position.  Temperature 0 is greedy decoding:
// d_j is accepted iff it equals the verifier's argmax, and the token after
// the accepted drafts is that argmax.
//
// Sequences of one cache advance together, so the step emits
// n = 1 + min_b r_b tokens for every sequence (r_b = accepted drafts of
// sequence b): for a sequence that accepted more, token n - 1 is its own
// accepted draft, itself a valid sample.
//
// Two kernels, one block per sequence each: spec_rows finds r_b,
// spec_finish emits the tokens and sets the cache length to n_0 + n.
#include "common.cuh"

namespace dory {

namespace {

constexpr int kSpecThreads = 256;

// Block maximum of v (all threads get it); red: 32 floats.
__device__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float m = -INFINITY;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  return m;
}

// Softmax numerator exp((z - zmax) * inv_t) of row z and its total over V.
__device__ void row_softmax_total(const float* z, int V, float inv_t,
                                  float* zmax_out, float* total_out,
                                  float* red) {
  float m = -INFINITY;
  for (int i = threadIdx.x; i < V; i += blockDim.x) m = fmaxf(m, z[i]);
  m = block_max(m, red);
  float s = 0.f;
  for (int i = threadIdx.x; i < V; i += blockDim.x) s += __expf((z[i] - m) * inv_t);
  s = block_sum(s, red);
  __syncthreads();
  *zmax_out = m;
  *total_out = s;
}

__global__ void __launch_bounds__(kSpecThreads)
spec_rows_kernel(SpecArgs a) {
  __shared__ float red[32];
  const int b = blockIdx.x, G1 = a.gamma + 1;
  const int* drf = a.draft + (size_t)b * G1;
  pdl_wait();
  pdl_trigger();
  int r = 0;
  if (a.inv_temp == 0.f) {
    const int* tgt = a.target + (size_t)b * G1;
    while (r < a.gamma && drf[r + 1] == tgt[r]) ++r;
  } else {
    for (; r < a.gamma; ++r) {
      const float* z = a.logits + ((size_t)b * G1 + r) * a.V;
      float zm, tot;
      row_softmax_total(z, a.V, a.inv_temp, &zm, &tot, red);
      const int d = drf[r + 1];
      const float p = (d >= 0 && d < a.V) ? __expf((z[d] - zm) * a.inv_temp) / tot
                                          : 0.f;
      if (!(a.uniform[(size_t)b * G1 + r] < p)) break;
    }
  }
  if (threadIdx.x == 0) a.r[b] = r;
}

// Inverse-CDF draw from weights w(x) = exp((z_x - zmax) * inv_t) over
// x != excl (excl < 0: none), with u in [0, 1).  Each thread owns a
// contiguous chunk of the vocabulary; an exclusive scan of the chunk totals
// locates the chunk that holds u * total, whose owner walks it.
__device__ int sample_row(const float* z, int V, float inv_t, int excl, float u,
                          float* red, float* pre, int* pick) {
  float zm, tot0;
  row_softmax_total(z, V, inv_t, &zm, &tot0, red);
  const int nt = blockDim.x, t = threadIdx.x;
  const int per = (V + nt - 1) / nt;
  const int lo = min(V, t * per), hi = min(V, lo + per);
  float s = 0.f;
  for (int i = lo; i < hi; ++i)
    if (i != excl) s += __expf((z[i] - zm) * inv_t);
  pre[t] = s;
  if (t == 0) *pick = -1;
  __syncthreads();
  if (t == 0) {                      // exclusive scan of nt totals
    float acc = 0.f;
    for (int i = 0; i < nt; ++i) {
      const float v = pre[i];
      pre[i] = acc;
      acc += v;
    }
    pre[nt] = acc;
  }
  __syncthreads();
  const float target = u * pre[nt];
  const float base = pre[t];
  if (hi > lo && base <= target && (target < base + s || t == nt - 1)) {
    float acc = base;
    int last = -1;
    for (int i = lo; i < hi; ++i) {
      if (i == excl) continue;
      last = i;
      acc += __expf((z[i] - zm) * inv_t);
      if (acc > target) break;
    }
    if (last >= 0) atomicMax(pick, last);
  }
  __syncthreads();
  int x = *pick;
  if (x < 0) {                       // rounding at the very top: last token
    x = (V - 1 == excl) ? V - 2 : V - 1;
  }
  return x;
}

__global__ void __launch_bounds__(kSpecThreads)
spec_finish_kernel(SpecArgs a) {
  __shared__ float red[32];
  __shared__ float pre[kSpecThreads + 1];
  __shared__ int pick;
  const int b = blockIdx.x, G1 = a.gamma + 1;
  const int* drf = a.draft + (size_t)b * G1;
  int* out = a.out + (size_t)b * G1;
  pdl_wait();
  pdl_trigger();
  int n = a.gamma;                   // accepted drafts, minimum over rows
  for (int i = 0; i < a.B; ++i) n = min(n, a.r[i]);
  for (int i = threadIdx.x; i < G1; i += blockDim.x)
    out[i] = i < n ? drf[i + 1] : -1;
  int tok;
  if (a.inv_temp == 0.f) {
    tok = a.target[(size_t)b * G1 + n];
  } else if (a.r[b] > n) {
    tok = drf[n + 1];                // this row accepted its draft here
  } else {
    const float* z = a.logits + ((size_t)b * G1 + n) * a.V;
    const int excl = n < a.gamma ? drf[n + 1] : -1;
    tok = sample_row(z, a.V, a.inv_temp, excl,
                     a.uniform[(size_t)b * G1 + a.gamma], red, pre, &pick);
  }
  if (threadIdx.x == 0) {
    out[n] = tok;
    if (b == 0) {
      *a.n_out = n + 1;
      *a.n_ctx = a.n0 + n + 1;
    }
  }
}

// [G1][B] (step-major draft tokens) -> [B][G1].
__global__ void spec_transpose_kernel(const int* src, int* dst, int B, int G1) {
  pdl_wait();
  pdl_trigger();
  for (int i = threadIdx.x; i < B * G1; i += blockDim.x) {
    const int j = i / B, b = i - j * B;
    dst[b * G1 + j] = src[i];
  }
}

}  // namespace

void launch_spec_accept(const SpecArgs& a, cudaStream_t st) {
  launch_k(spec_rows_kernel, dim3(a.B), dim3(kSpecThreads), 0, st, a);
  launch_k(spec_finish_kernel, dim3(a.B), dim3(kSpecThreads), 0, st, a);
}

void launch_spec_transpose(const int* src, int* dst, int B, int G1,
                           cudaStream_t st) {
  launch_k(spec_transpose_kernel, dim3(1), dim3(256), 0, st, src, dst, B, G1);
}

}  // namespace dory
