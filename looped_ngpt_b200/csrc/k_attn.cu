// Prefill attention (T query tokens per sequence) over the paged / ring KV
// cache; decode (one token) is in k_attn_decode.cu.
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
#include "warp_mma.cuh"

namespace dory {

namespace {

constexpr int TK = 64;          // keys per shared-memory tile
constexpr int KPAD = 8;         // bf16 padding per K/V row (bank spread)

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

// --------------------------------------------------------------- prefill --
// grid (ceil(T/64), Hq, B); block 256 = 64 query rows x 4 threads.
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

void launch_attn_prefill(const AttnArgs& a, cudaStream_t st) {
  switch (a.dm.hd) {
    case 64: launch_prefill_t<64>(a, st); break;
    case 128: launch_prefill_t<128>(a, st); break;
    default: launch_prefill_t<160>(a, st); break;
  }
}

}  // namespace dory
