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
// One warp: sum the split-K partials of one head of the fused QKVG output,
// rotate (rotate-half RoPE), L2-normalise over the head, scale per dim.
// Writes the head to dst (f32); `round` keeps only BF16 precision (the value
// the cache will hold for this token).
__device__ __forceinline__ void head_rope_norm(const float* src, size_t pstride,
                                               int S, int col0, int hd,
                                               const float* rope,
                                               const float* scale,
                                               float extra, bool round,
                                               float* dst) {
  const int lane = threadIdx.x & 31, half = hd / 2;
  constexpr int kPairs = kMaxHeadDim / 64;
  float r1[kPairs], r2[kPairs];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < kPairs; ++j) {
    const int i = lane + 32 * j;
    r1[j] = r2[j] = 0.f;
    if (i < half) {
      float x1 = 0.f, x2 = 0.f;
      for (int s = 0; s < S; ++s) {
        x1 += src[s * pstride + col0 + i];
        x2 += src[s * pstride + col0 + i + half];
      }
      const float c = rope[2 * i], sn = rope[2 * i + 1];
      r1[j] = x1 * c - x2 * sn;
      r2[j] = x2 * c + x1 * sn;
      ss += r1[j] * r1[j] + r2[j] * r2[j];
    }
  }
  const float inv = 1.f / fmaxf(sqrtf(warp_sum(ss)), 1e-12f);
#pragma unroll
  for (int j = 0; j < kPairs; ++j) {
    const int i = lane + 32 * j;
    if (i < half) {
      float a = r1[j] * inv * scale[i] * extra;
      float b = r2[j] * inv * scale[i + half] * extra;
      if (round) {
        a = __bfloat162float(__float2bfloat16_rn(a));
        b = __bfloat162float(__float2bfloat16_rn(b));
      }
      dst[i] = a;
      dst[i + half] = b;
    }
  }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   (uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}

// Issue cp.async copies of keys/values [j0, j0 + nk) of (b, kvh) into shared
// rows, skipping position `skip` (the current token, filled from registers
// later).  Row addresses: ring slots or 64-token pages, no division.
template <int HD>
__device__ __forceinline__ void issue_kv_tile(bf16* Ks, bf16* Vs,
                                              const KVSlot& kv,
                                              const CacheGeo& g, int Hkv,
                                              int b, int kvh, int j0, int nk,
                                              int skip, int NT) {
  constexpr int VEC = HD / 8;
  constexpr int RP = HD + KPAD;
  const int ring_slot0 = kv.ring ? j0 % kv.cap : 0;
  for (int id = threadIdx.x; id < nk * VEC; id += NT) {
    const int r = id / VEC, c = id - r * VEC;      // VEC is a constant
    const int j = j0 + r;
    if (j == skip) continue;
    size_t off;
    if (kv.ring) {
      int slot = ring_slot0 + r;
      if (slot >= kv.cap) slot -= kv.cap;
      off = ((size_t)(b * Hkv + kvh) * kv.cap + slot) * HD;
    } else {
      const int page = g.block_table[b * g.pages_per_seq + (j >> 6)];
      off = (((size_t)page * Hkv + kvh) * kPage + (j & 63)) * HD;
    }
    cp_async16(Ks + r * RP + c * 8, kv.K + off + c * 8);
    cp_async16(Vs + r * RP + c * 8, kv.V + off + c * 8);
  }
}

// grid (kMaxSplits, Hkv, B); block NT = 2 * HD threads.  One query token per
// sequence; G query heads share the KV head.  Each block:
//   (0) before the dependency wait, starts copying the cached keys/values of
//       its first tile (positions < p were written by finished calls);
//   (1) forms q for its G query heads and the new k, v of its KV head from
//       the QKVG partials (RoPE, per-head L2 norm, scales);
//   (2) the block whose key range ends at p stores k, v in the cache;
//   (3) attends over its key range in tiles of 64 keys (position p from
//       shared memory): scores split HD/32 ways per key, probabilities by
//       one warp per head, P.V split over 4 key groups;
//   (4) writes its partial (m, l, o); (5) takes a ticket -- the last block
//       of (b, kvh) merges all splits, applies sigmoid(gate), writes the
//       bf16 head outputs and resets the ticket counter to 0.
// No block waits on another.
template <int HD, int G>
__global__ void __launch_bounds__(2 * HD) attn_decode_fused_kernel(const DecAttnArgs a) {
  constexpr int NT = 2 * HD;
  constexpr int NQ = HD / 32;          // score parts per key
  constexpr int RP = HD + KPAD;
  constexpr int HP = HD / 2;           // dim pairs
  // P.V partials, later the merge's weights and gates
  constexpr int PVS = (4 * G * HD > G * (2 * kMaxSplits + HD))
                          ? 4 * G * HD : G * (2 * kMaxSplits + HD);
  // splits staged per merge round trip: as many as fit in the K/V tiles
  constexpr int CHF = (2 * TK * (HD + KPAD) * 2) / (G * HD * 4);
  constexpr int CH = CHF < 16 ? CHF : 16;
  static_assert(CH >= 1, "merge staging buffer must fit in the K/V tiles");
  extern __shared__ float sm[];
  const Dims& dm = a.dm;
  const int b = blockIdx.z, kvh = blockIdx.y, split = blockIdx.x;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;

  float* q_s = sm;                                   // [G][HD]
  float* kn_s = q_s + G * HD;                        // [HD]
  float* vn_s = kn_s + HD;                           // [HD]
  float* sc_s = vn_s + HD;                           // [NQ][G][TK] scores / [G][TK] probs
  float* st = sc_s + NQ * G * TK;                    // m, l, corr: [3][G] (+pad)
  float* pv_s = st + 32;                             // [4][G][HD] P.V partials
  bf16* K_s = reinterpret_cast<bf16*>(pv_s + PVS);   // [TK][RP]
  bf16* V_s = K_s + TK * RP;
  __shared__ int s_last;

  const int p = *a.g.n_ctx;
  const Split sp = split_of(p, a.window);
  const bool active = split < sp.n && p < a.g.max_ctx;
  const int k_begin = sp.lo + split * sp.chunk;
  const int k_end = min(sp.hi, k_begin + sp.chunk);
  if (active)
    issue_kv_tile<HD>(K_s, V_s, a.kv, a.g, dm.Hkv, b, kvh, k_begin,
                      min(TK, k_end - k_begin), p, NT);
  asm volatile("cp.async.commit_group;" ::: "memory");
  pdl_wait();
  pdl_trigger();
  if (!active) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (p >= a.g.max_ctx && split == 0 && tid == 0) atomicOr(a.err, ERRBIT_BOUNDS);
    return;
  }

  // (1) q heads, new k and v
  const float* src = a.qkvg + (size_t)b * dm.rows_qkvg;
  const size_t pstride = (size_t)a.B * dm.rows_qkvg;
  for (int item = w; item < G + 2; item += NT / 32) {
    if (item < G) {
      const int h = kvh * G + item;
      head_rope_norm(src, pstride, a.S, h * HD, HD, a.rope, a.s_q + h * HD,
                     a.q_scale, false, q_s + item * HD);
    } else if (item == G) {
      head_rope_norm(src, pstride, a.S, dm.qdim + kvh * HD, HD, a.rope,
                     a.s_k + kvh * HD, 1.f, true, kn_s);
    } else {
      for (int c = lane; c < HD; c += 32) {
        float v = 0.f;
        for (int s2 = 0; s2 < a.S; ++s2)
          v += src[s2 * pstride + dm.qdim + dm.kvdim + kvh * HD + c];
        vn_s[c] = __bfloat162float(__float2bfloat16_rn(v));
      }
    }
  }
  if (tid < G) { st[tid] = -INFINITY; st[G + tid] = 0.f; }
  __syncthreads();

  // (2) the block whose range ends at p stores the new entry
  if (k_end == p + 1) {
    const size_t off = kv_index(a.kv, a.g, dm.Hkv, HD, b, kvh, p);
    for (int c = tid; c < HD; c += NT) {
      a.kv.K[off + c] = __float2bfloat16_rn(kn_s[c]);
      a.kv.V[off + c] = __float2bfloat16_rn(vn_s[c]);
    }
  }

  // (3) tiles
  float acc[G][2];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g][0] = acc[g][1] = 0.f;
  const int dp = tid % HP, kg = tid / HP;            // P.V: dim pair, key group
  for (int j0 = k_begin; j0 < k_end; j0 += TK) {
    const int nk = min(TK, k_end - j0);
    if (j0 != k_begin) {
      __syncthreads();                               // previous tile consumed
      issue_kv_tile<HD>(K_s, V_s, a.kv, a.g, dm.Hkv, b, kvh, j0, nk, p, NT);
      asm volatile("cp.async.commit_group;" ::: "memory");
    }
    if (p >= j0 && p < j0 + nk) {                    // current token's row
      for (int c = tid; c < HD; c += NT) {
        K_s[(p - j0) * RP + c] = __float2bfloat16_rn(kn_s[c]);
        V_s[(p - j0) * RP + c] = __float2bfloat16_rn(vn_s[c]);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    {   // scores: thread -> (key j, 32-dim part qp)
      const int j = tid % TK, qp = tid / TK;
      float sg[G];
#pragma unroll
      for (int g = 0; g < G; ++g) sg[g] = 0.f;
      if (j < nk) {
        const bf16* kk = K_s + j * RP + qp * 32;
#pragma unroll
        for (int c = 0; c < 32; c += 8) {
          const uint4 kv = *reinterpret_cast<const uint4*>(kk + c);
          const float k0 = bf_lo(kv.x), k1 = bf_hi(kv.x), k2 = bf_lo(kv.y),
                      k3 = bf_hi(kv.y), k4 = bf_lo(kv.z), k5 = bf_hi(kv.z),
                      k6 = bf_lo(kv.w), k7 = bf_hi(kv.w);
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float* qq = q_s + g * HD + qp * 32 + c;
            const float4 qa = *reinterpret_cast<const float4*>(qq);
            const float4 qb = *reinterpret_cast<const float4*>(qq + 4);
            float t = sg[g];
            t = fmaf(qa.x, k0, t); t = fmaf(qa.y, k1, t);
            t = fmaf(qa.z, k2, t); t = fmaf(qa.w, k3, t);
            t = fmaf(qb.x, k4, t); t = fmaf(qb.y, k5, t);
            t = fmaf(qb.z, k6, t); t = fmaf(qb.w, k7, t);
            sg[g] = t;
          }
        }
      }
#pragma unroll
      for (int g = 0; g < G; ++g) sc_s[(qp * G + g) * TK + j] = sg[g];
    }
    __syncthreads();
    if (w < G) {   // probabilities of head w over this tile
      float s0 = -INFINITY, s1 = -INFINITY;
      if (lane < nk) {
        s0 = 0.f;
        for (int q = 0; q < NQ; ++q) s0 += sc_s[(q * G + w) * TK + lane];
      }
      if (lane + 32 < nk) {
        s1 = 0.f;
        for (int q = 0; q < NQ; ++q) s1 += sc_s[(q * G + w) * TK + lane + 32];
      }
      const float m_old = st[w];
      const float m_new = fmaxf(m_old, warp_max(fmaxf(s0, s1)));
      const float e0 = exp2f(s0 - m_new), e1 = exp2f(s1 - m_new);
      __syncwarp();
      sc_s[w * TK + lane] = e0;                      // row w of [G][TK]
      sc_s[w * TK + lane + 32] = e1;
      const float sum = warp_sum(e0 + e1);
      if (lane == 0) {
        const float corr = exp2f(m_old - m_new);
        st[2 * G + w] = corr;
        st[G + w] = st[G + w] * corr + sum;
        st[w] = m_new;
      }
    }
    __syncthreads();
    {   // P.V over this tile: thread -> (dim pair dp, keys [16 kg, 16 kg + 16))
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float c = st[2 * G + g];
        acc[g][0] *= c;
        acc[g][1] *= c;
      }
      const int jb = kg * 16, je = min(nk, jb + 16);
      for (int j = jb; j < je; ++j) {
        const float2 v = __bfloat1622float2(
            *reinterpret_cast<const __nv_bfloat162*>(V_s + j * RP + 2 * dp));
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float pg = sc_s[g * TK + j];
          acc[g][0] = fmaf(pg, v.x, acc[g][0]);
          acc[g][1] = fmaf(pg, v.y, acc[g][1]);
        }
      }
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    pv_s[(kg * G + g) * HD + 2 * dp] = acc[g][0];
    pv_s[(kg * G + g) * HD + 2 * dp + 1] = acc[g][1];
  }
  __syncthreads();

  // (4) partial of this split
  const size_t hb = (size_t)b * dm.Hq + kvh * G;
  for (int idx = tid; idx < G * HD; idx += NT) {
    const int g = idx / HD, c = idx - g * HD;
    const float o = pv_s[(0 * G + g) * HD + c] + pv_s[(1 * G + g) * HD + c] +
                    pv_s[(2 * G + g) * HD + c] + pv_s[(3 * G + g) * HD + c];
    a.part_o[((hb + g) * kMaxSplits + split) * HD + c] = o;
  }
  if (tid < G) {
    float* ml = a.part_ml + ((hb + tid) * kMaxSplits + split) * 2;
    ml[0] = st[tid];
    ml[1] = st[G + tid];
  }

  // (5) ticket; the last block of (b, kvh) merges the splits
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    int* cnt = a.counters + b * dm.Hkv + kvh;
    s_last = (atomicAdd(cnt, 1) == sp.n - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // merge: stage (m, l) of every split and the gate sums in one round trip
  float* mlw = pv_s;                                 // [G][n][2] (n <= 64)
  float* gate_s = pv_s + G * kMaxSplits * 2;         // [G][HD]
  for (int id = tid; id < G * sp.n; id += NT) {
    const int g = id / sp.n, s2 = id - g * sp.n;
    const float2 v = __ldcg(reinterpret_cast<const float2*>(
        a.part_ml + ((hb + g) * kMaxSplits + s2) * 2));
    mlw[2 * id] = v.x;
    mlw[2 * id + 1] = v.y;
  }
  for (int idx = tid; idx < G * HD; idx += NT) {
    const int g = idx / HD, c = idx - g * HD;
    float gs = 0.f;
    for (int s3 = 0; s3 < a.S; ++s3)
      gs += src[s3 * pstride + dm.qdim + 2 * dm.kvdim + (kvh * G + g) * HD + c];
    gate_s[idx] = sigmoidf_(gs);
  }
  __syncthreads();
  if (w < G) {
    float M = -INFINITY;
    for (int s2 = lane; s2 < sp.n; s2 += 32) M = fmaxf(M, mlw[2 * (w * sp.n + s2)]);
    M = warp_max(M);
    float L = 0.f;
    for (int s2 = lane; s2 < sp.n; s2 += 32) {
      const int id = w * sp.n + s2;
      const float f = exp2f(mlw[2 * id] - M);
      mlw[2 * id] = f;                               // merge weight of split
      L += f * mlw[2 * id + 1];
    }
    L = warp_sum(L);
    if (lane == 0) st[w] = 1.f / L;
  }
  // partial outputs, CH splits per round trip, staged with cp.async
  constexpr int NO = (G * HD + NT - 1) / NT;         // outputs per thread
  float* buf = reinterpret_cast<float*>(K_s);        // [G][CH][HD]
  float o[NO];
#pragma unroll
  for (int k = 0; k < NO; ++k) o[k] = 0.f;
  for (int s0 = 0; s0 < sp.n; s0 += CH) {
    const int cnt = min(CH, sp.n - s0);
    __syncthreads();                                 // buf free, weights ready
    constexpr int V4 = HD / 4;                       // 16-byte pieces per row
    for (int id = tid; id < G * cnt * V4; id += NT) {
      const int row = id / V4, c = id - row * V4;
      const int g = row / cnt, s2 = row - g * cnt;
      cp_async16(buf + (g * CH + s2) * HD + c * 4,
                 a.part_o + ((hb + g) * kMaxSplits + s0 + s2) * HD + c * 4);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
#pragma unroll
    for (int k = 0; k < NO; ++k) {
      const int idx = tid + k * NT;
      if (idx < G * HD) {
        const int g = idx / HD, c = idx - g * HD;
        const float* f = mlw + 2 * (g * sp.n + s0);
        float t = o[k];
        for (int s2 = 0; s2 < cnt; ++s2)
          t = fmaf(f[2 * s2], buf[(g * CH + s2) * HD + c], t);
        o[k] = t;
      }
    }
  }
#pragma unroll
  for (int k = 0; k < NO; ++k) {
    const int idx = tid + k * NT;
    if (idx < G * HD) {
      const int g = idx / HD, c = idx - g * HD;
      a.a_out[(size_t)b * dm.qdim + (kvh * G + g) * HD + c] =
          __float2bfloat16_rn(gate_s[idx] * o[k] * st[g]);
    }
  }
  if (tid == 0) a.counters[b * dm.Hkv + kvh] = 0;
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
  pdl_wait();
  pdl_trigger();
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
  launch_k(attn_prefill_kernel<HD>, grid, dim3(256), smem, st, a);
}

}  // namespace

template <int HD, int G>
void launch_dec_t(const DecAttnArgs& a, cudaStream_t st) {
  constexpr int NQ = HD / 32;
  constexpr int PVS = (4 * G * HD > G * (2 * kMaxSplits + HD))
                          ? 4 * G * HD : G * (2 * kMaxSplits + HD);
  const size_t smem = (G * HD + 2 * HD + NQ * G * TK + 32 + PVS) *
                          sizeof(float) +
                      2 * TK * (HD + KPAD) * sizeof(bf16);
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(attn_decode_fused_kernel<HD, G>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    configured = true;
  }
  launch_k(attn_decode_fused_kernel<HD, G>, dim3(kMaxSplits, a.dm.Hkv, a.B),
           dim3(2 * HD), smem, st, a);
}

template <int HD>
void launch_dec_hd(const DecAttnArgs& a, cudaStream_t st) {
  switch (a.dm.Hq / a.dm.Hkv) {
    case 1: launch_dec_t<HD, 1>(a, st); break;
    case 2: launch_dec_t<HD, 2>(a, st); break;
    case 4: launch_dec_t<HD, 4>(a, st); break;
    default: launch_dec_t<HD, 8>(a, st); break;
  }
}

void launch_attn_decode_fused(const DecAttnArgs& a, cudaStream_t st) {
  switch (a.dm.hd) {
    case 64: launch_dec_hd<64>(a, st); break;
    case 128: launch_dec_hd<128>(a, st); break;
    default: launch_dec_hd<160>(a, st); break;
  }
}

void launch_attn_prefill(const AttnArgs& a, cudaStream_t st) {
  switch (a.dm.hd) {
    case 64: launch_prefill_t<64>(a, st); break;
    case 128: launch_prefill_t<128>(a, st); break;
    default: launch_prefill_t<160>(a, st); break;
  }
}

}  // namespace dory
