// GQA attention over the paged / ring KV cache.
//
// Visible keys for a query at position p: j <= p, and for sliding-window
// layers additionally j > p - W (W = 1024 for Dory; the paper summary,
// 技术新颖性: 3:1 sliding-window to full attention).  Query head h reads KV
// head h / (Hq / Hkv).  Scores use exp2: q arrives pre-multiplied by
// sqrt(head_dim) * log2(e), so exp2(q.k - m) is the softmax numerator.
// The gate sigmoid(g) multiplies the head outputs; the L2 norm of the gated
// concatenation that precedes W_o (paperlayer §2) is folded into the
// normalised update that follows W_o (N(W N(a)) = N(W a)).
#include "common.cuh"

namespace dory {

namespace {

constexpr int TK = 64;          // keys per shared-memory tile
constexpr int KPAD = 8;         // bf16 padding per K/V row (bank spread)

// Key range [lo, hi) of a query at position p, and the split of that range
// into at most kMaxSplits chunks of a multiple of TK keys.
struct Split {
  int lo, hi, chunk, n;
};
__device__ __forceinline__ Split split_of(int p, int window) {
  Split s;
  s.lo = window ? max(0, p - window + 1) : 0;
  s.hi = p + 1;
  const int nk = s.hi - s.lo;
  int c = (nk + kMaxSplits - 1) / kMaxSplits;
  c = ((c + TK - 1) / TK) * TK;
  s.chunk = c;
  s.n = (nk + c - 1) / c;
  return s;
}

// Copy keys [j0, j0 + nk) of (b, kvh) into shared rows [0, nk).
__device__ __forceinline__ void load_tile(bf16* dst, const bf16* base,
                                          const KVSlot& kv, const CacheGeo& g,
                                          int Hkv, int hd, int b, int kvh,
                                          int j0, int nk) {
  const int vec = hd / 8;
  for (int id = threadIdx.x; id < nk * vec; id += blockDim.x) {
    const int r = id / vec, c = id - r * vec;
    const size_t off = kv_index(kv, g, Hkv, hd, b, kvh, j0 + r);
    *reinterpret_cast<uint4*>(dst + r * (hd + KPAD) + c * 8) =
        *reinterpret_cast<const uint4*>(base + off + c * 8);
  }
}

// ---------------------------------------------------------------- decode --
// grid (kMaxSplits, Hkv, B); block 256.  One query per sequence (T = 1).
__global__ void __launch_bounds__(256) attn_decode_kernel(const AttnArgs a) {
  extern __shared__ float sm[];
  const Dims& dm = a.dm;
  const int hd = dm.hd, G = dm.Hq / dm.Hkv;
  const int b = blockIdx.z, kvh = blockIdx.y, split = blockIdx.x;
  const int p = *a.g.n_ctx;
  const Split sp = split_of(p, a.window);
  if (split >= sp.n) return;
  if (p >= a.g.max_ctx) return;   // reported by the K/V writer
  const int k_begin = sp.lo + split * sp.chunk;
  const int k_end = min(sp.hi, k_begin + sp.chunk);

  float* q_s = sm;                                   // [G][hd]
  float* p_s = q_s + G * hd;                         // [G][TK]
  float* st = p_s + G * TK;                          // m, l, corr: [3][G]
  bf16* K_s = reinterpret_cast<bf16*>(st + 3 * 16);  // [TK][hd + KPAD]
  bf16* V_s = K_s + TK * (hd + KPAD);

  const float* qsrc = a.q + (size_t)b * dm.qdim + kvh * G * hd;
  for (int i = threadIdx.x; i < G * hd; i += blockDim.x) q_s[i] = qsrc[i];
  if (threadIdx.x < G) { st[threadIdx.x] = -INFINITY; st[G + threadIdx.x] = 0.f; }

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;

  for (int j0 = k_begin; j0 < k_end; j0 += TK) {
    const int nk = min(TK, k_end - j0);
    __syncthreads();
    load_tile(K_s, a.kv.K, a.kv, a.g, dm.Hkv, hd, b, kvh, j0, nk);
    load_tile(V_s, a.kv.V, a.kv, a.g, dm.Hkv, hd, b, kvh, j0, nk);
    __syncthreads();
    for (int pr = threadIdx.x; pr < G * TK; pr += blockDim.x) {
      const int gg = pr / TK, j = pr - gg * TK;
      float s = -INFINITY;
      if (j < nk) {
        const float* qq = q_s + gg * hd;
        const bf16* kk = K_s + j * (hd + KPAD);
        float acc2 = 0.f;
        for (int c = 0; c < hd; c += 8) {
          const uint4 kv = *reinterpret_cast<const uint4*>(kk + c);
          acc2 = fmaf(qq[c + 0], bf_lo(kv.x), acc2);
          acc2 = fmaf(qq[c + 1], bf_hi(kv.x), acc2);
          acc2 = fmaf(qq[c + 2], bf_lo(kv.y), acc2);
          acc2 = fmaf(qq[c + 3], bf_hi(kv.y), acc2);
          acc2 = fmaf(qq[c + 4], bf_lo(kv.z), acc2);
          acc2 = fmaf(qq[c + 5], bf_hi(kv.z), acc2);
          acc2 = fmaf(qq[c + 6], bf_lo(kv.w), acc2);
          acc2 = fmaf(qq[c + 7], bf_hi(kv.w), acc2);
        }
        s = acc2;
      }
      p_s[pr] = s;
    }
    __syncthreads();
    if (w < G) {
      const float s0 = p_s[w * TK + lane], s1 = p_s[w * TK + lane + 32];
      const float m_old = st[w];
      const float m_new = fmaxf(m_old, warp_max(fmaxf(s0, s1)));
      const float e0 = exp2f(s0 - m_new), e1 = exp2f(s1 - m_new);
      p_s[w * TK + lane] = e0;
      p_s[w * TK + lane + 32] = e1;
      const float sum = warp_sum(e0 + e1);
      if (lane == 0) {
        const float corr = exp2f(m_old - m_new);
        st[2 * G + w] = corr;
        st[G + w] = st[G + w] * corr + sum;
        st[w] = m_new;
      }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int idx = threadIdx.x + r * 256;
      if (idx < G * hd) {
        const int gg = idx / hd, c = idx - gg * hd;
        float v = acc[r] * st[2 * G + gg];
        const float* pp = p_s + gg * TK;
        for (int j = 0; j < nk; ++j)
          v = fmaf(pp[j], __bfloat162float(V_s[j * (hd + KPAD) + c]), v);
        acc[r] = v;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int idx = threadIdx.x + r * 256;
    if (idx < G * hd) {
      const int gg = idx / hd, c = idx - gg * hd;
      const int h = kvh * G + gg;
      a.part_o[(((size_t)b * dm.Hq + h) * kMaxSplits + split) * hd + c] = acc[r];
    }
  }
  if (threadIdx.x < G) {
    const int h = kvh * G + threadIdx.x;
    float* ml = a.part_ml + (((size_t)b * dm.Hq + h) * kMaxSplits + split) * 2;
    ml[0] = st[threadIdx.x];
    ml[1] = st[G + threadIdx.x];
  }
}

// grid (Hq, B); block hd.  Merge the splits, apply the gate, emit bf16.
__global__ void attn_combine_kernel(const AttnArgs a) {
  const Dims& dm = a.dm;
  const int h = blockIdx.x, b = blockIdx.y, c = threadIdx.x;
  const int p = *a.g.n_ctx;
  const Split sp = split_of(p, a.window);
  const size_t base = ((size_t)b * dm.Hq + h) * kMaxSplits;
  float M = -INFINITY;
  for (int s = 0; s < sp.n; ++s) M = fmaxf(M, a.part_ml[(base + s) * 2]);
  float L = 0.f, o = 0.f;
  for (int s = 0; s < sp.n; ++s) {
    const float f = exp2f(a.part_ml[(base + s) * 2] - M);
    L += f * a.part_ml[(base + s) * 2 + 1];
    o += f * a.part_o[(base + s) * dm.hd + c];
  }
  const size_t oi = (size_t)b * dm.qdim + h * dm.hd + c;
  a.a_out[oi] = __float2bfloat16_rn(a.gate[oi] * (o / L));
}

// --------------------------------------------------------------- prefill --
// grid (ceil(T/64), Hq, B); block 256 = 64 query rows x 4 threads.
template <int HD>
__global__ void __launch_bounds__(256) attn_prefill_kernel(const AttnArgs a) {
  constexpr int QP = HD + 4;           // padded f32 row of Q
  constexpr int KP = HD + KPAD;        // padded bf16 row of K / V
  constexpr int DQ = HD / 4;           // output dims per thread
  extern __shared__ float sm[];
  float* Q_s = sm;                                   // [64][QP]
  float* P_s = Q_s + 64 * QP;                        // [64][TK]
  bf16* K_s = reinterpret_cast<bf16*>(P_s + 64 * TK);
  bf16* V_s = K_s + TK * KP;
  const Dims& dm = a.dm;
  const int G = dm.Hq / dm.Hkv;
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / G;
  const int t0 = blockIdx.x * 64;
  const int r = threadIdx.x >> 2, qc = threadIdx.x & 3;
  const int n0 = *a.g.n_ctx;
  const int t = t0 + r;
  const bool valid = t < a.T;
  const int p = n0 + t;
  if (n0 + a.T > a.g.max_ctx) return;   // reported by the K/V writer

  for (int i = threadIdx.x; i < 64 * HD; i += 256) {
    const int rr = i / HD, c = i - rr * HD;
    float v = 0.f;
    if (t0 + rr < a.T) v = a.q[((size_t)b * a.T + t0 + rr) * dm.qdim + h * HD + c];
    Q_s[rr * QP + c] = v;
  }
  const int kmin = a.window ? max(0, n0 + t0 - a.window + 1) : 0;
  const int kmax = n0 + min(a.T, t0 + 64);
  float m = -INFINITY, l = 0.f;
  float acc[DQ];
#pragma unroll
  for (int i = 0; i < DQ; ++i) acc[i] = 0.f;

  for (int j0 = kmin; j0 < kmax; j0 += TK) {
    const int nk = min(TK, kmax - j0);
    __syncthreads();
    load_tile(K_s, a.kv.K, a.kv, a.g, dm.Hkv, HD, b, kvh, j0, nk);
    load_tile(V_s, a.kv.V, a.kv, a.g, dm.Hkv, HD, b, kvh, j0, nk);
    __syncthreads();
    float s[16];
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int jj = qc + 4 * i, j = j0 + jj;
      const bool vis = valid && jj < nk && j <= p && (!a.window || j > p - a.window);
      float v = -INFINITY;
      if (vis) {
        const float* qq = Q_s + r * QP;
        const bf16* kk = K_s + jj * KP;
        float d0 = 0.f;
#pragma unroll 4
        for (int c = 0; c < HD; c += 8) {
          const uint4 kv = *reinterpret_cast<const uint4*>(kk + c);
          const float4 qa = *reinterpret_cast<const float4*>(qq + c);
          const float4 qb = *reinterpret_cast<const float4*>(qq + c + 4);
          d0 = fmaf(qa.x, bf_lo(kv.x), d0);
          d0 = fmaf(qa.y, bf_hi(kv.x), d0);
          d0 = fmaf(qa.z, bf_lo(kv.y), d0);
          d0 = fmaf(qa.w, bf_hi(kv.y), d0);
          d0 = fmaf(qb.x, bf_lo(kv.z), d0);
          d0 = fmaf(qb.y, bf_hi(kv.z), d0);
          d0 = fmaf(qb.z, bf_lo(kv.w), d0);
          d0 = fmaf(qb.w, bf_hi(kv.w), d0);
        }
        v = d0;
      }
      s[i] = v;
      mx = fmaxf(mx, v);
    }
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    float corr = 1.f, sum = 0.f;
    if (m_new != -INFINITY) {
      corr = exp2f(m - m_new);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float e = exp2f(s[i] - m_new);
        P_s[r * TK + qc + 4 * i] = e;
        sum += e;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) P_s[r * TK + qc + 4 * i] = 0.f;
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    l = l * corr + sum;
    m = m_new;
    __syncwarp();
#pragma unroll
    for (int i = 0; i < DQ; ++i) acc[i] *= corr;
    for (int jj = 0; jj < nk; ++jj) {
      const float pv = P_s[r * TK + jj];
      const bf16* vv = V_s + jj * KP + qc * DQ;
#pragma unroll
      for (int i = 0; i < DQ; i += 2) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vv + i));
        acc[i] = fmaf(pv, f.x, acc[i]);
        acc[i + 1] = fmaf(pv, f.y, acc[i + 1]);
      }
    }
  }
  if (!valid) return;
  const float inv = 1.f / l;
  const size_t row = (size_t)b * a.T + t;
#pragma unroll
  for (int i = 0; i < DQ; ++i) {
    const size_t oi = row * dm.qdim + h * HD + qc * DQ + i;
    a.a_out[oi] = __float2bfloat16_rn(a.gate[oi] * acc[i] * inv);
  }
}

template <int HD>
void launch_prefill_t(const AttnArgs& a, cudaStream_t st) {
  const size_t smem = (64 * (HD + 4) + 64 * TK) * sizeof(float) +
                      2 * TK * (HD + KPAD) * sizeof(bf16);
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(attn_prefill_kernel<HD>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    configured = true;
  }
  dim3 grid((a.T + 63) / 64, a.dm.Hq, a.B);
  attn_prefill_kernel<HD><<<grid, 256, smem, st>>>(a);
}

}  // namespace

void launch_attn_decode(const AttnArgs& a, cudaStream_t st) {
  const int hd = a.dm.hd, G = a.dm.Hq / a.dm.Hkv;
  const size_t smem = (G * hd + G * TK + 48) * sizeof(float) +
                      2 * TK * (hd + KPAD) * sizeof(bf16);
  static size_t configured = 0;
  if (smem > 48 * 1024 && smem > configured) {
    cudaFuncSetAttribute(attn_decode_kernel,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    configured = smem;
  }
  dim3 grid(kMaxSplits, a.dm.Hkv, a.B);
  attn_decode_kernel<<<grid, 256, smem, st>>>(a);
}

void launch_attn_combine(const AttnArgs& a, cudaStream_t st) {
  dim3 grid(a.dm.Hq, a.B);
  attn_combine_kernel<<<grid, a.dm.hd, 0, st>>>(a);
}

void launch_attn_prefill(const AttnArgs& a, cudaStream_t st) {
  switch (a.dm.hd) {
    case 64: launch_prefill_t<64>(a, st); break;
    case 128: launch_prefill_t<128>(a, st); break;
    default: launch_prefill_t<160>(a, st); break;
  }
}

}  // namespace dory
