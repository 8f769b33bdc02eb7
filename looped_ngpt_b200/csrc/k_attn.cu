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
  constexpr int CHF = (4 * TK * (HD + KPAD) * 2) / (G * HD * 4);
  constexpr int CH = CHF < 32 ? CHF : 32;
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
  bf16* Kb = reinterpret_cast<bf16*>(pv_s + PVS);    // [2][TK][RP]
  bf16* Vb = Kb + 2 * TK * RP;                       // [2][TK][RP]
  bf16* K_s = Kb;                                    // merge staging base
  __shared__ int s_last;

  const int p = *a.g.n_ctx;
  const Split sp = split_of(p, a.window);
  const bool active = split < sp.n && p < a.g.max_ctx;
  const int k_begin = sp.lo + split * sp.chunk;
  const int k_end = min(sp.hi, k_begin + sp.chunk);
  if (active)
    issue_kv_tile<HD>(Kb, Vb, a.kv, a.g, dm.Hkv, b, kvh, k_begin,
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
  // tiles are double-buffered: tile it + 1 is in flight while tile it is
  // consumed, tile it + 2 is issued once tile it's buffer is free
  if (k_begin + TK < k_end) {
    issue_kv_tile<HD>(Kb + TK * RP, Vb + TK * RP, a.kv, a.g, dm.Hkv, b, kvh,
                      k_begin + TK, min(TK, k_end - k_begin - TK), p, NT);
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  int it = 0;
  for (int j0 = k_begin; j0 < k_end; j0 += TK, ++it) {
    const int nk = min(TK, k_end - j0);
    bf16* K_s = Kb + (it & 1) * TK * RP;
    bf16* V_s = Vb + (it & 1) * TK * RP;
    if (p >= j0 && p < j0 + nk) {                    // current token's row
      for (int c = tid; c < HD; c += NT) {
        K_s[(p - j0) * RP + c] = __float2bfloat16_rn(kn_s[c]);
        V_s[(p - j0) * RP + c] = __float2bfloat16_rn(vn_s[c]);
      }
    }
    if (j0 + TK < k_end) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else asm volatile("cp.async.wait_group 0;" ::: "memory");
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
    if (j0 + 2 * TK < k_end) {
      __syncthreads();                               // tile it's buffer is free
      issue_kv_tile<HD>(K_s, V_s, a.kv, a.g, dm.Hkv, b, kvh, j0 + 2 * TK,
                        min(TK, k_end - j0 - 2 * TK), p, NT);
      asm volatile("cp.async.commit_group;" ::: "memory");
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
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0,
                                        uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0,
                                          uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile(
      "ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
      : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
      : "r"(addr));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4],
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Flash attention for prefill (T query tokens per sequence), one query head
// per block, 64 queries (4 warps x 16 rows) per block, 64-key tiles of the
// head's KV cache double-buffered in shared memory with cp.async.  S = Q K^T
// and O += P V on the warp-level tensor-core path (m16n8k16, bf16 operands,
// f32 accumulation); P stays in registers between the two products; online
// softmax in exp2 units (q is pre-scaled by sqrt(h) log2 e).  Causal and
// sliding-window masks per element.  Epilogue: gate * O / l as bf16.
// grid (ceil(T/64), Hq, B); block 128.
template <int HD>
__global__ void __launch_bounds__(128) attn_prefill_kernel(const AttnArgs a) {
  constexpr int RP = HD + KPAD;
  constexpr int KS = HD / 16;        // k-steps of Q K^T
  constexpr int NO = HD / 8;         // n-tiles of O
  extern __shared__ __align__(16) uint8_t smraw[];
  bf16* Ks = reinterpret_cast<bf16*>(smraw);          // [2][64][RP]
  bf16* Vs = Ks + 2 * 64 * RP;                        // [2][64][RP]
  const Dims& dm = a.dm;
  const int G = dm.Hq / dm.Hkv;
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / G;
  const int t0 = blockIdx.x * 64;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, tq = lane & 3;

  // finite contents everywhere (partial tiles leave rows unwritten)
  for (int i = threadIdx.x; i < 4 * 64 * RP / 8; i += 128)
    reinterpret_cast<uint4*>(smraw)[i] = make_uint4(0, 0, 0, 0);
  pdl_wait();
  pdl_trigger();
  const int n0 = *a.g.n_ctx;
  if (n0 + a.T > a.g.max_ctx) return;                 // reported by the writer

  const int tr0 = t0 + 16 * warp + g, tr1 = tr0 + 8;  // call-local rows
  const int p0 = n0 + tr0, p1 = n0 + tr1;             // positions
  uint32_t qf[KS][4];
  {
    const bf16* q0 = a.q + ((size_t)b * a.T + min(tr0, a.T - 1)) * dm.qdim + h * HD;
    const bf16* q1 = a.q + ((size_t)b * a.T + min(tr1, a.T - 1)) * dm.qdim + h * HD;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      const int c = 16 * kk + 2 * tq;
      qf[kk][0] = *reinterpret_cast<const uint32_t*>(q0 + c);
      qf[kk][1] = *reinterpret_cast<const uint32_t*>(q1 + c);
      qf[kk][2] = *reinterpret_cast<const uint32_t*>(q0 + c + 8);
      qf[kk][3] = *reinterpret_cast<const uint32_t*>(q1 + c + 8);
    }
  }
  float o[NO][4];
#pragma unroll
  for (int n = 0; n < NO; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;

  const int kmin = a.window ? max(0, n0 + t0 - a.window + 1) : 0;
  const int kmax = n0 + min(a.T, t0 + 64);
  __syncthreads();                                    // zero fill done
  issue_kv_tile<HD>(Ks, Vs, a.kv, a.g, dm.Hkv, b, kvh, kmin,
                    min(64, kmax - kmin), -1, 128);
  asm volatile("cp.async.commit_group;" ::: "memory");
  const uint32_t ks0 = (uint32_t)__cvta_generic_to_shared(Ks);
  const uint32_t vs0 = (uint32_t)__cvta_generic_to_shared(Vs);

  int it = 0;
  for (int j0 = kmin; j0 < kmax; j0 += 64, ++it) {
    const int buf = it & 1;
    if (j0 + 64 < kmax) {
      issue_kv_tile<HD>(Ks + (buf ^ 1) * 64 * RP, Vs + (buf ^ 1) * 64 * RP,
                        a.kv, a.g, dm.Hkv, b, kvh, j0 + 64,
                        min(64, kmax - j0 - 64), -1, 128);
      asm volatile("cp.async.commit_group;" ::: "memory");
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const uint32_t kb = ks0 + buf * 64 * RP * 2, vb = vs0 + buf * 64 * RP * 2;

    // S = Q K^T, 8 n-tiles of 8 keys
    float sc[8][4];
#pragma unroll
    for (int n = 0; n < 8; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
      for (int nj = 0; nj < 4; ++nj) {
        const int key = 16 * nj + (lane & 7) + ((lane >> 4) << 3);
        const int col = 16 * kk + ((lane >> 3) & 1) * 8;
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kb + (key * RP + col) * 2, b0, b1, b2, b3);
        mma16816(sc[2 * nj], qf[kk], b0, b1);
        mma16816(sc[2 * nj + 1], qf[kk], b2, b3);
      }
    }
    // masks and online softmax (rows r0 = g, r1 = g + 8 of this warp)
    float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int j = j0 + 8 * n + 2 * tq + e;
        const bool in = j < kmax;
        const bool v0 = in && j <= p0 && (!a.window || j > p0 - a.window);
        const bool v1 = in && j <= p1 && (!a.window || j > p1 - a.window);
        if (!v0) sc[n][e] = -INFINITY;
        if (!v1) sc[n][2 + e] = -INFINITY;
        mx0 = fmaxf(mx0, sc[n][e]);
        mx1 = fmaxf(mx1, sc[n][2 + e]);
      }
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float ref0 = mn0 == -INFINITY ? 0.f : mn0;   // all masked so far
    const float ref1 = mn1 == -INFINITY ? 0.f : mn1;
    const float c0 = exp2f(m0 - ref0), c1 = exp2f(m1 - ref1);
    float s0 = 0.f, s1 = 0.f;
    uint32_t pf[4][4];                                // P as A fragments
#pragma unroll
    for (int n = 0; n < 8; ++n) {
      const float e0 = exp2f(sc[n][0] - ref0), e1 = exp2f(sc[n][1] - ref0);
      const float e2 = exp2f(sc[n][2] - ref1), e3 = exp2f(sc[n][3] - ref1);
      s0 += e0 + e1;
      s1 += e2 + e3;
      const int kk2 = n >> 1, hi = n & 1;
      pf[kk2][hi * 2 + 0] = pack_bf16(e0, e1);
      pf[kk2][hi * 2 + 1] = pack_bf16(e2, e3);
    }
    s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
    s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
    s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
    l0 = l0 * c0 + s0;
    l1 = l1 * c1 + s1;
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int n = 0; n < NO; ++n) {
      o[n][0] *= c0; o[n][1] *= c0;
      o[n][2] *= c1; o[n][3] *= c1;
    }
    // O += P V: 4 k-steps of 16 keys, NO/2 pairs of 8-dim n-tiles
#pragma unroll
    for (int kk2 = 0; kk2 < 4; ++kk2) {
      const uint32_t af[4] = {pf[kk2][0], pf[kk2][1], pf[kk2][2], pf[kk2][3]};
#pragma unroll
      for (int nn = 0; nn < NO / 2; ++nn) {
        const int key = 16 * kk2 + (lane & 15);
        const int col = 16 * nn + ((lane >> 4) << 3);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vb + (key * RP + col) * 2, b0, b1, b2, b3);
        mma16816(o[2 * nn], af, b0, b1);
        mma16816(o[2 * nn + 1], af, b2, b3);
      }
    }
    __syncthreads();                                  // buffer free for reuse
  }

  // epilogue: a = gate * O / l
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
#pragma unroll
  for (int n = 0; n < NO; ++n) {
    const int dim = h * HD + 8 * n + 2 * tq;
    if (tr0 < a.T) {
      const size_t r = ((size_t)b * a.T + tr0) * dm.qdim + dim;
      const float2 gv = *reinterpret_cast<const float2*>(a.gate + r);
      *reinterpret_cast<__nv_bfloat162*>(a.a_out + r) =
          __floats2bfloat162_rn(gv.x * o[n][0] * i0, gv.y * o[n][1] * i0);
    }
    if (tr1 < a.T) {
      const size_t r = ((size_t)b * a.T + tr1) * dm.qdim + dim;
      const float2 gv = *reinterpret_cast<const float2*>(a.gate + r);
      *reinterpret_cast<__nv_bfloat162*>(a.a_out + r) =
          __floats2bfloat162_rn(gv.x * o[n][2] * i1, gv.y * o[n][3] * i1);
    }
  }
}

template <int HD>
void launch_prefill_t(const AttnArgs& a, cudaStream_t st) {
  const size_t smem = 4 * 64 * (HD + KPAD) * sizeof(bf16);
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(attn_prefill_kernel<HD>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    configured = true;
  }
  dim3 grid((a.T + 63) / 64, a.dm.Hq, a.B);
  launch_k(attn_prefill_kernel<HD>, grid, dim3(128), smem, st, a);
}

}  // namespace

template <int HD, int G>
void launch_dec_t(const DecAttnArgs& a, cudaStream_t st) {
  constexpr int NQ = HD / 32;
  constexpr int PVS = (4 * G * HD > G * (2 * kMaxSplits + HD))
                          ? 4 * G * HD : G * (2 * kMaxSplits + HD);
  const size_t smem = (G * HD + 2 * HD + NQ * G * TK + 32 + PVS) *
                          sizeof(float) +
                      4 * TK * (HD + KPAD) * sizeof(bf16);
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
