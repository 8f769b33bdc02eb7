// Prefill attention (T query tokens per sequence) on the sm_100a tensor
// cores: flash attention with S = Q K^T and O += P V as tcgen05 MMAs into
// tensor memory, operands staged by TMA.
//
// Visible keys for a query at position p: j <= p, and for sliding-window
// layers also j > p - W (W = 1024 for Dory; the paper summary, 技术新颖性:
// 3:1 sliding-window to full attention).  Query head h reads KV head h / G.
// q arrives pre-multiplied by sqrt(head_dim) * log2(e), so the softmax
// numerator is exp2(s - m).  The gate sigmoid(g) multiplies the head outputs;
// the L2 norm of the gated concatenation before W_o (paperlayer §2) is folded
// into the normalised update after W_o (N(W N(a)) = N(W a)).  The call's own
// keys and values are already in the cache (written by the QKV projection),
// so every query reads keys from one place.
//
// One CTA = 128 queries of one head (grid (ceil(T / 128), Hq, B), longest key
// ranges first) against 64-key tiles of the head's KV cache.  Operands live
// in shared memory as 64-dim panels with the 128-byte swizzle plus, for
// head_dim % 64 == 32, a 32-dim panel with the 64-byte swizzle.  Six warps:
//   warp 0 lane 0   TMA: the Q tile once, then K and V tiles through a
//                   3-stage ring (a 64-key tile is one 64-token page or one
//                   64-slot run of a ring, whose capacity is a multiple of 64);
//                   a stage's K slot is refilled as soon as S = Q K^T has
//                   read it, its V slot once O += P V has;
//   warp 1 lane 0   MMA: S_j = Q K_j^T (M 128, N 64, K 16 per instruction)
//                   into one of two TMEM S buffers, then, once the softmax
//                   has written P_j, O += P_j V_j (V as the MN-major B
//                   operand) into the TMEM O accumulator; S_{j+1} is issued
//                   before O += P_j V_j so the softmax of j+1 overlaps it;
//   warps 2-9       softmax, two warps per TMEM lane quarter: the thread of
//                   query row r in warp half c takes keys 32c..32c+31 of
//                   each tile (its TMEM lane, one 32-column load); the two
//                   halves exchange row maxima through shared memory; running
//                   max m and sums l; O is rescaled in TMEM (each half its
//                   own 32-column chunks) only when m grows by more than 2^8
//                   (P stays <= 2^8 otherwise, and O / l is exact for any
//                   common m); P as bf16 into the shared-memory A operand;
//                   finally O / l times the gate, as bf16.
// Every mbarrier wait is bounded: a timeout sets ERRBIT_TIMEOUT; the CTA
// waits (bounded) for its copies and MMAs, frees TMEM and exits.
#include "async_copy.cuh"
#include "common.cuh"
#include "tcgen05.cuh"
#include "warp_mma.cuh"

#include <cstdio>

namespace dory {

namespace {

constexpr int PQ = 128;                 // queries per CTA (TMEM lanes)
constexpr int PK = 64;                  // keys per tile
constexpr int PST = 3;                  // K/V stages
constexpr int kSmWarps = 8;             // softmax warps (2 per lane quarter)
constexpr int kPfThreads = (2 + kSmWarps) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr int NSB = 3;                  // TMEM S buffers (S issued 2 tiles ahead)
constexpr uint32_t kOCol = NSB * PK;    // O accumulator after the S buffers
constexpr float kHeadroom = 8.f;        // log2 growth of m before O rescales

// Shared-memory operand of `rows` rows x HD dims: N128 panels of 64 dims
// (rows x 128 B, 128-byte swizzle) then N64 panels of 32 dims (rows x 64 B,
// 64-byte swizzle).
template <int HD>
struct PfOp {
  static constexpr int N128 = HD / 64, N64 = (HD % 64) / 32;
  static_assert(HD % 32 == 0, "head_dim must be a multiple of 32");
  static constexpr int bytes(int rows) { return rows * (128 * N128 + 64 * N64); }
  static constexpr int Q = bytes(PQ), KV = bytes(PK);
  static constexpr int STAGE = 2 * KV;                 // K tile, then V tile
  static constexpr int P = PQ * PK * 2;                // one 64-key panel
  static constexpr int SMEM = 1024 + Q + PST * STAGE + 2 * P;   // P double-buffered
  static constexpr int KS = HD / 16;                   // k-steps of Q K^T
};

struct PfMaps {
  CUtensorMap q128, q64, k128, k64, v128, v64;
};

// Descriptor of k-step kk (16 dims) of a K-major [rows x HD] operand.
template <int HD>
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t base, int rows, int kk) {
  using L = PfOp<HD>;
  if (kk < 4 * L::N128)
    return make_sdesc(base + (kk >> 2) * rows * 128 + (kk & 3) * 32, 16, 1024, kSw128);
  return make_sdesc(base + L::N128 * rows * 128 + (kk - 4 * L::N128) * 32, 16, 512,
                    kSw64);
}

// 2^x on the SFU (one instruction; flushes subnormal results to zero, and
// exp2(-inf) = 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// First row of the 64-key tile t of (b, kvh) in the [rows][hd] cache view.
__device__ __forceinline__ int pf_tile_row(const KVSlot& kv, const CacheGeo& g,
                                           int Hkv, int b, int kvh, int t) {
  const int j = t * PK;
  if (kv.ring) return (b * Hkv + kvh) * kv.cap + j % kv.cap;
  const int page = g.block_table[b * g.pages_per_seq + j / kPage];
  return (page * Hkv + kvh) * kPage;
}

template <int HD>
__global__ void __launch_bounds__(kPfThreads, 1)
attn_prefill_tc_kernel(const __grid_constant__ PfMaps mp, const AttnArgs a) {
  using L = PfOp<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (su32(smem_raw) & 1023)) & 1023);
  uint8_t* sQ = base;
  uint8_t* sKV = base + L::Q;
  uint8_t* sP = sKV + PST * L::STAGE;
  // K and V slots of a stage fill and free separately: K_j is free once
  // S_j = Q K_j^T completes, V_j once O += P_j V_j completes
  __shared__ __align__(8) uint64_t q_full, k_full[PST], k_empty[PST], v_full[PST],
      v_empty[PST];
  // indexed so that no barrier can run two phases ahead of its waiter:
  //   s_full / s_free[j % NSB] (phase j / NSB): S buffer filled / read;
  //   p_full[j & 1] (phase j >> 1): P buffer written;
  //   o_done[j & 1] (phase j >> 1): O += P_j V_j complete (and all before it)
  __shared__ __align__(8) uint64_t s_full[NSB], s_free[NSB], p_full[2], o_done[2],
      mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ int s_fail, s_issued_k, s_issued_v;
  __shared__ float xch[2][PQ];                      // row max / sum exchange
  volatile int* fail = &s_fail;

  const Dims& dm = a.dm;
  const int G = dm.Hq / dm.Hkv;
  const int qt = gridDim.x - 1 - blockIdx.x;         // longest ranges first
  const int h = blockIdx.y, b = blockIdx.z, kvh = h / G;
  const int q0 = qt * PQ;                            // call-local first row
  const int nq = min(PQ, a.T - q0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(&q_full, 1);
    for (int i = 0; i < PST; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(k_empty + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(v_empty + i, 1);
    }
    for (int i = 0; i < NSB; ++i) {
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, kSmWarps);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(p_full + i, kSmWarps);
      mbar_init(o_done + i, 1);
    }
    mbar_init(&mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_fail = 0;
    s_issued_k = 0;
    s_issued_v = 0;
  }
  if (warp == 0) tmem_alloc(&tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  pdl_wait();
  pdl_trigger();

  // query positions [plo, phi] of the valid rows; key tiles [t_lo, t_lo + nkt)
  const int n0 = *a.g.n_ctx;
  const int plo = n0 + q0, phi = n0 + q0 + nq - 1;
  const int klo = a.window ? max(0, plo - a.window + 1) : 0;
  const int t_lo = klo / PK;
  const int nkt = n0 + a.T <= a.g.max_ctx ? phi / PK - t_lo + 1 : 0;

  if (warp == 0) {
    // ---- TMA producer ----------------------------------------------------
    if (lane == 0 && nkt > 0) {
      const int qrow = b * a.T + q0;
      mbar_expect_tx(&q_full, L::Q);
      for (int i = 0; i < L::N128; ++i)
        tma_load_2d(sQ + i * PQ * 128, &mp.q128, h * HD + 64 * i, qrow, &q_full);
      if (L::N64)
        tma_load_2d(sQ + L::N128 * PQ * 128, &mp.q64, h * HD + 64 * L::N128, qrow,
                    &q_full);
      // K tiles run up to PST ahead of V tiles; both wait (non-blocking
      // checks, bounded in total) for their slot of PST tiles earlier
      auto load = [&](int jt, bool is_v) {
        const int s = jt % PST;
        const int row = pf_tile_row(a.kv, a.g, dm.Hkv, b, kvh, t_lo + jt);
        uint8_t* dst = sKV + s * L::STAGE + (is_v ? L::KV : 0);
        uint64_t* bar = (is_v ? v_full : k_full) + s;
        const CUtensorMap* m128 = is_v ? &mp.v128 : &mp.k128;
        const CUtensorMap* m64 = is_v ? &mp.v64 : &mp.k64;
        mbar_expect_tx(bar, L::KV);
        for (int i = 0; i < L::N128; ++i) tma_load_2d(dst + i * PK * 128, m128, 64 * i, row, bar);
        if (L::N64) tma_load_2d(dst + L::N128 * PK * 128, m64, 64 * L::N128, row, bar);
      };
      int jk = 0, jv = 0;
      long idle = 0;
      while (jv < nkt && !*fail) {
        bool did = false;
        if (jk < nkt &&
            (jk < PST || mbar_try(k_empty + jk % PST, (uint32_t)((jk / PST - 1) & 1)))) {
          load(jk++, false);
          s_issued_k = jk;
          did = true;
        }
        if (jv < jk &&
            (jv < PST || mbar_try(v_empty + jv % PST, (uint32_t)((jv / PST - 1) & 1)))) {
          load(jv++, true);
          s_issued_v = jv;
          did = true;
        }
        if (did) idle = 0;
        else if (++idle > kSpin) {
          atomicOr(&s_fail, 1);
          break;
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer --------------------------------------------------------
    if (lane == 0 && nkt > 0) {
      constexpr uint32_t id_s = idesc_bf16(PQ, PK);
      constexpr uint32_t id_o128 = idesc_bf16(PQ, 64 * L::N128, true);
      constexpr uint32_t id_o64 = idesc_bf16(PQ, 32, true);
      const uint32_t q_s = su32(sQ), p_s = su32(sP);
      bool ok = mbar_wait(&q_full, 0);
      auto issue_s = [&](int j) {
        const int s = j % PST, bb = j % NSB;
        if (!mbar_wait(k_full + s, (uint32_t)((j / PST) & 1)) ||
            (j >= NSB && !mbar_wait(s_free + bb, (uint32_t)((j / NSB - 1) & 1))))
          return false;
        tc_fence_after();
        const uint32_t k_s = su32(sKV + s * L::STAGE);
#pragma unroll
        for (int kk = 0; kk < L::KS; ++kk)
          umma_bf16(tmem + bb * PK, kmajor_desc<HD>(q_s, PQ, kk),
                    kmajor_desc<HD>(k_s, PK, kk), id_s, kk > 0);
        umma_commit(k_empty + s);             // K_j read
        umma_commit(s_full + bb);
        return true;
      };
      auto issue_pv = [&](int j) {
        const int s = j % PST;
        if (!mbar_wait(p_full + (j & 1), (uint32_t)((j >> 1) & 1)) ||
            !mbar_wait(v_full + s, (uint32_t)((j / PST) & 1)))
          return false;
        tc_fence_after();
        const uint32_t v_s = su32(sKV + s * L::STAGE + L::KV);
        const uint32_t pj = p_s + (j & 1) * L::P;
#pragma unroll
        for (int kk = 0; kk < PK / 16; ++kk) {
          const uint64_t pa = make_sdesc(pj + kk * 32, 16, 1024, kSw128);
          // V rows are keys (K); 16 keys = two 8-row groups
          umma_bf16(tmem + kOCol, pa,
                    make_sdesc(v_s + kk * 2048, PK * 128, 1024, kSw128), id_o128,
                    (j | kk) != 0);
          if (L::N64)
            umma_bf16(tmem + kOCol + 64 * L::N128, pa,
                      make_sdesc(v_s + L::N128 * PK * 128 + kk * 1024, PK * 64, 512,
                                 kSw64),
                      id_o64, (j | kk) != 0);
        }
        umma_commit(v_empty + s);             // V_j read
        umma_commit(o_done + (j & 1));        // O holds P_0 V_0 + .. + P_j V_j
        return true;
      };
      // S runs NSB - 1 tiles ahead of O += P V, so the softmax of tile j + 1
      // never waits for its scores behind O += P_j V_j
      for (int j = 0; ok && j < NSB - 1 && j < nkt; ++j) ok = issue_s(j);
      for (int j = 0; ok && j < nkt; ++j)
        ok = (j + NSB - 1 >= nkt || issue_s(j + NSB - 1)) && issue_pv(j);
      if (!ok) atomicOr(&s_fail, 1);
      umma_commit(&mma_done);
    }
  } else {
    // ---- softmax and epilogue: thread = query row = TMEM lane ------------
    const int qw = warp & 3, hf = (warp - 2) >> 2;  // lane quarter, key half
    const int row = 32 * qw + lane;
    const int pos = n0 + q0 + row;
    const uint32_t trow = tmem + ((uint32_t)(32 * qw) << 16);
    // the two warps of a lane quarter: named barrier 1 + qw, 64 threads
    auto pair_sync = [&] {
      asm volatile("bar.sync %0, 64;" ::"r"(1 + qw) : "memory");
    };
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nkt; ++j) {
      const int bb = j % NSB;
      if (!mbar_wait_warp(s_full + bb, (uint32_t)((j / NSB) & 1))) { ok = false; break; }
      tc_fence_after();
      float sv[32];
      tmem_ld32(trow + bb * PK + 32 * hf, sv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_free + bb);
      const int k0 = (t_lo + j) * PK + 32 * hf;       // this half's first key
      float mt = -INFINITY;
      // whole half visible to every row of the CTA: no per-key test
      const bool inner = k0 + 31 <= plo && (!a.window || k0 > phi - a.window);
      if (inner) {
#pragma unroll
        for (int c = 0; c < 32; ++c) mt = fmaxf(mt, sv[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          const int key = k0 + c;
          const bool vis = key <= pos && (!a.window || key > pos - a.window);
          sv[c] = vis ? sv[c] : -INFINITY;
          mt = fmaxf(mt, sv[c]);
        }
      }
      xch[hf][row] = mt;
      pair_sync();
      mt = fmaxf(mt, xch[hf ^ 1][row]);
      const float m_new = fmaxf(m_ref, mt);
      const bool need = m_new > m_ref + kHeadroom;   // also -inf -> finite
      // O may be rescaled once P_{j-1} V_{j-1} is done (rare: m grew by
      // more than the headroom); P buffer j & 1 is free once P_{j-2} V_{j-2}
      // is done
      const bool resc = j > 0 && __any_sync(0xffffffffu, need);
      if (j >= 2 && !mbar_wait_warp(o_done + (j & 1), (uint32_t)(((j - 2) >> 1) & 1))) {
        ok = false;
        break;
      }
      if (resc && !mbar_wait_warp(o_done + ((j - 1) & 1), (uint32_t)(((j - 1) >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (resc) {
        const float f = need ? fast_exp2(m_ref - m_new) : 1.f;
#pragma unroll 1
        for (int c0 = 32 * hf; c0 < HD; c0 += 64) {
          float t[32];
          tmem_ld32(trow + kOCol + c0, t);
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) t[i2] *= f;
          tmem_st32(trow + kOCol + c0, t);
        }
        l *= f;
      }
      if (need) m_ref = m_new;
      // P row (bf16) into the 128-byte-swizzled A operand; four partial sums
      uint8_t* prow = sP + (j & 1) * L::P + row * 128;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      // a row with no visible key yet has m = -inf and only -inf scores
      const float msub = m_ref == -INFINITY ? 0.f : m_ref;
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        float e[8];
#pragma unroll
        for (int i2 = 0; i2 < 8; ++i2) {
          e[i2] = fast_exp2(sv[8 * c8 + i2] - msub);   // exp2(-inf) = 0
          ls[i2 & 3] += e[i2];
        }
        uint4 u;
        u.x = pack_bf16(e[0], e[1]);
        u.y = pack_bf16(e[2], e[3]);
        u.z = pack_bf16(e[4], e[5]);
        u.w = pack_bf16(e[6], e[7]);
        const int c = 4 * hf + c8;                    // 16-byte chunk of the row
        *reinterpret_cast<uint4*>(prow + ((c ^ (row & 7)) << 4)) = u;
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full + (j & 1));
    }
    if (!ok) atomicOr(&s_fail, 1);
    // epilogue: O / l times the gate (l summed over the two halves)
    // the last O += P V (the commit covers every MMA before it)
    const bool got = ok && nkt > 0 &&
                     mbar_wait_warp(o_done + ((nkt - 1) & 1), (uint32_t)(((nkt - 1) >> 1) & 1));
    xch[hf][row] = l;
    pair_sync();
    if (got) {
      tc_fence_after();
      const float lt = l + xch[hf ^ 1][row];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      const size_t r = (size_t)b * a.T + q0 + row;
#pragma unroll 1
      for (int c0 = 32 * hf; c0 < HD; c0 += 64) {
        float t[32];
        tmem_ld32(trow + kOCol + c0, t);
        if (row < nq) {
          const float* gr = a.gate + r * dm.qdim + h * HD + c0;
          bf16* dst = a.a_out + r * dm.qdim + h * HD + c0;
#pragma unroll
          for (int i2 = 0; i2 < 32; i2 += 2)
            *reinterpret_cast<__nv_bfloat162*>(dst + i2) = __floats2bfloat162_rn(
                t[i2] * inv * gr[i2], t[i2 + 1] * inv * gr[i2 + 1]);
        }
      }
    } else if (nkt > 0) {
      atomicOr(&s_fail, 1);
    }
  }

  // teardown: the MMAs (and after a failure the copies) must be complete
  // before shared memory and TMEM are released
  __syncthreads();
  if (threadIdx.x == 0 && nkt > 0) {
    if (!mbar_wait(&mma_done, 0)) atomicOr(&s_fail, 1);
    if (*fail) {
      atomicOr(a.err, ERRBIT_TIMEOUT);
      mbar_wait(&q_full, 0);
      for (int which = 0; which < 2; ++which) {
        const int hi = which ? s_issued_v : s_issued_k, lo = hi > PST ? hi - PST : 0;
        uint64_t* full = which ? v_full : k_full;
        for (int j = lo; j < hi; ++j)
          if (!mbar_wait(full + j % PST, (uint32_t)((j / PST) & 1))) break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_free(tmem, kTmemCols);
  }
}

template <int HD>
void launch_pf_t(const AttnArgs& a, const CUtensorMap* kv_maps, cudaStream_t st) {
  using L = PfOp<HD>;
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(attn_prefill_tc_kernel<HD>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
    configured = true;
  }
  PfMaps mp;
  const long M = (long)a.B * a.T;
  if (!make_act_map(&mp.q128, a.q, M, a.dm.qdim, 64, PQ) ||
      !make_act_map(&mp.q64, a.q, M, a.dm.qdim, 32, PQ)) {
    note_host_failure("prefill attention: tensor map");
    return;
  }
  mp.k128 = kv_maps[0];
  mp.k64 = kv_maps[1];
  mp.v128 = kv_maps[2];
  mp.v64 = kv_maps[3];
  dim3 grid((a.T + PQ - 1) / PQ, a.dm.Hq, a.B);
  launch_k(attn_prefill_tc_kernel<HD>, grid, dim3(kPfThreads), (size_t)L::SMEM, st,
           mp, a);
}

}  // namespace

int pf_tile_keys() { return PK; }

void launch_attn_prefill_tc(const AttnArgs& a, const CUtensorMap* kv_maps,
                            cudaStream_t st) {
  switch (a.dm.hd) {
    case 64: launch_pf_t<64>(a, kv_maps, st); break;
    case 128: launch_pf_t<128>(a, kv_maps, st); break;
    default: launch_pf_t<160>(a, kv_maps, st); break;
  }
}

}  // namespace dory
