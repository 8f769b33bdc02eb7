// BF16 GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA) for prefill
// projections: C[M, N] = A[M, K] * W[N, K]^T (f32 accumulate), A the bf16
// activations (row stride lda), W the bf16 weights, both K-contiguous.
//
// Persistent CTAs (one per SM at most) walk 128 x 256 output tiles:
//   warp 0 lane 0  streams 128x64 A and 256x64 W tiles with 2-D TMA loads
//                  (128-byte swizzle) into a ring of STAGES shared-memory
//                  stages (full/empty mbarriers), across tile boundaries;
//   warp 1 lane 0  issues tcgen05.mma.cta_group::1.kind::f16 (M=128, N=256,
//                  K=16; 4 per stage) into one of two 256-column f32 TMEM
//                  accumulators and releases each stage with tcgen05.commit;
//   warps 2-5      wait for a finished accumulator, read it with tcgen05.ld
//                  (warp w owns TMEM lanes 32 (w % 4) .. + 31 = tile rows),
//                  run the epilogue (f32 store, optional per-column scale,
//                  the SwiGLU pairing of gate/up column halves, or the QKV
//                  head epilogue) and hand the buffer back to the MMA warp,
//                  so epilogues overlap the next tile's MMAs.
// Every mbarrier wait is bounded: on timeout the CTA records ERRBIT_TIMEOUT,
// waits (bounded) for its outstanding copies and MMAs, frees TMEM and exits.
//
// Many-row plain and SwiGLU GEMMs (prefill) run on CTA pairs instead
// (gemm_tc_pair_kernel below: clusters of two, tcgen05 cta_group::2,
// 256 x 256 tiles, each CTA staging its own A rows and half of the W rows),
// which cuts by a third the shared-memory operand traffic per FLOP that
// limits the one-CTA tile.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <map>
#include <mutex>
#include <utility>

#include "async_copy.cuh"
#include "common.cuh"
#include "tcgen05.cuh"

namespace dory {

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr uint32_t kStageA = BM * BK * 2;     // 16 KB
constexpr uint32_t kStageB = BN * BK * 2;     // 32 KB
// Shared-memory matrix descriptor of a K-major tile stored by TMA with the
// 128-byte swizzle: rows of 64 bf16 (128 B), 8-row atoms 1024 B apart.
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr) {
  return make_sdesc(saddr, 16, 1024, kSw128);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

enum TcMode : int { TC_PLAIN = 0, TC_SWIGLU = 1, TC_QKV = 2 };

struct TcArgs {
  int M, N, K;          // output rows, output columns (SwiGLU: features)
  int up_off;           // SwiGLU: row offset of the up half of W
  float* C;             // TC_PLAIN: f32 out [M][ldc]
  bf16* Cb;             // TC_SWIGLU: bf16 out [M][ldc]
  int ldc;
  long slab;            // TC_PLAIN with K splits: elements between partials
  const float* col_scale;
  const float* out_scale;   // scalar factor on every product (NVFP4 tensor
                            // scale of dequantised weights), or null
  int* err;
  // TC_QKV: one tile column = one head of the fused q/k/v/gate projection
  int T;                // tokens per sequence (rows are b * T + t)
  int Hq, Hkv, qdim, kvdim;
  const float* s_q; const float* s_k;
  const float* rope;    // this layer type's table [T][hd/2][2] (cos, sin)
  float q_scale;
  KVSlot kv; CacheGeo g;
  bf16* q_out;          // [M][qdim] bf16, scaled by sqrt(hd) log2 e
  float* gate_out;      // [M][qdim] sigmoid(gate)
  const int* row_loops; // rows with their own loop counts, or null
  int loop_t;           // loop of this layer pass (0: non-recurrent)
};

// Epilogue of a TC_QKV tile: this thread holds one row of one head (hd
// columns).  q/k: rotate-half RoPE at the row's position, L2 norm over the
// head, per-dim scale; k and v go to the KV cache slot, q to q_out; gate
// heads get the sigmoid.
template <int HD>
__device__ __forceinline__ void qkv_epilogue(const TcArgs& a, int item,
                                             int row, float (&v)[HD]) {
  const int b = row / a.T, t = row - b * a.T;
  int kind, head, col0;
  if (item < a.Hq) { kind = 0; head = item; col0 = head * HD; }
  else if (item < a.Hq + a.Hkv) { kind = 1; head = item - a.Hq; col0 = a.qdim + head * HD; }
  else if (item < a.Hq + 2 * a.Hkv) {
    kind = 2; head = item - a.Hq - a.Hkv; col0 = a.qdim + a.kvdim + head * HD;
  } else {
    kind = 3; head = item - a.Hq - 2 * a.Hkv; col0 = a.qdim + 2 * a.kvdim + head * HD;
  }
  (void)col0;
  if (kind == 3) {
    float* dst = a.gate_out + (size_t)row * a.qdim + head * HD;
#pragma unroll
    for (int i = 0; i < HD; i += 4)
      *reinterpret_cast<float4*>(dst + i) =
          make_float4(sigmoidf_(v[i]), sigmoidf_(v[i + 1]), sigmoidf_(v[i + 2]),
                      sigmoidf_(v[i + 3]));
    return;
  }
  const int p = *a.g.n_ctx + t;
  if (kind != 0 && p >= a.g.max_ctx) {
    atomicOr(a.err, ERRBIT_BOUNDS);
    return;
  }
  // a row that sits out this loop writes no K/V
  if (kind != 0 && !row_writes_kv(a.row_loops, b, a.loop_t)) return;
  if (kind != 2) {
    constexpr int H2 = HD / 2;
    const float* rt = a.rope + (size_t)t * H2 * 2;
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < H2; ++i) {
      const float2 cs = *reinterpret_cast<const float2*>(rt + 2 * i);
      const float x1 = v[i], x2 = v[i + H2];
      v[i] = x1 * cs.x - x2 * cs.y;
      v[i + H2] = x2 * cs.x + x1 * cs.y;
      ss += v[i] * v[i] + v[i + H2] * v[i + H2];
    }
    const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
    const float* sc = (kind == 0 ? a.s_q : a.s_k) + head * HD;
    const float f = kind == 0 ? inv * a.q_scale : inv;
#pragma unroll
    for (int i = 0; i < HD; ++i) v[i] *= sc[i] * f;
  }
  bf16* dst;
  if (kind == 0) dst = a.q_out + (size_t)row * a.qdim + head * HD;
  else dst = (kind == 1 ? a.kv.K : a.kv.V) +
             kv_index(a.kv, a.g, a.Hkv, HD, b, head, p);
#pragma unroll
  for (int i = 0; i < HD; i += 8) {
    uint4 u;
    u.x = pack2(v[i], v[i + 1]); u.y = pack2(v[i + 2], v[i + 3]);
    u.z = pack2(v[i + 4], v[i + 5]); u.w = pack2(v[i + 6], v[i + 7]);
    *reinterpret_cast<uint4*>(dst + i) = u;
  }
}

// Epilogue of one output row of a tile: this thread owns TMEM lane `trow`
// (row `row` of C), columns n0 .. of the tile (column tile ni, K split z).
template <int MODE, int TN>
__device__ __forceinline__ void epilogue_row(const TcArgs& a, uint32_t trow,
                                             int row, int n0, int ni, int z) {
  constexpr int OUTC = MODE == TC_SWIGLU ? TN / 2 : TN;   // output columns
  if (MODE == TC_PLAIN) {
    for (int c0 = 0; c0 < TN; c0 += 32) {
      float v[32];
      tmem_ld32(trow + c0, v);
      if (a.out_scale) {
        const float os = *a.out_scale;
#pragma unroll
        for (int k = 0; k < 32; ++k) v[k] *= os;
      }
      const int col = n0 + c0;
      if (row < a.M && col < a.N) {
        float* dst = a.C + z * a.slab + (size_t)row * a.ldc + col;
        if (a.col_scale) {
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (col + k < a.N) v[k] *= a.col_scale[col + k];
        }
        // 16-byte stores only when every row start stays 16-byte aligned
        if (col + 32 <= a.N && (a.ldc & 3) == 0) {
#pragma unroll
          for (int k = 0; k < 32; k += 4)
            *reinterpret_cast<float4*>(dst + k) =
                make_float4(v[k], v[k + 1], v[k + 2], v[k + 3]);
        } else {
          for (int k = 0; k < 32 && col + k < a.N; ++k) dst[k] = v[k];
        }
      }
    }
  } else if (MODE == TC_SWIGLU) {
    for (int c0 = 0; c0 < TN / 2; c0 += 32) {
      float gt[32], u[32];
      tmem_ld32(trow + c0, gt);
      tmem_ld32(trow + TN / 2 + c0, u);
      if (a.out_scale) {
        const float os = *a.out_scale;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          gt[k] *= os;
          u[k] *= os;
        }
      }
      const int col = n0 + c0;
      // columns of this tile only (TN / 2 need not be a multiple of 32)
      const int lim = min(32, min(OUTC - c0, a.N - col));
      if (row < a.M && lim > 0) {
        bf16* dst = a.Cb + (size_t)row * a.ldc + col;
        if (lim == 32 && (a.ldc & 1) == 0) {
#pragma unroll
          for (int k = 0; k < 32; k += 2)
            *reinterpret_cast<__nv_bfloat162*>(dst + k) = __floats2bfloat162_rn(
                gt[k] * sigmoidf_(gt[k]) * u[k],
                gt[k + 1] * sigmoidf_(gt[k + 1]) * u[k + 1]);
        } else {
          // unrolled with a predicate so that gt and u stay in registers
#pragma unroll
          for (int k = 0; k < 32; ++k)
            if (k < lim) dst[k] = __float2bfloat16_rn(gt[k] * sigmoidf_(gt[k]) * u[k]);
        }
      }
    }
  } else {
    float v[TN];
#pragma unroll
    for (int c0 = 0; c0 < TN; c0 += 32) {
      float t32[32];
      tmem_ld32(trow + c0, t32);
#pragma unroll
      for (int k = 0; k < 32; ++k) v[c0 + k] = t32[k];
    }
    if (a.out_scale) {
      const float os = *a.out_scale;
#pragma unroll
      for (int k = 0; k < TN; ++k) v[k] *= os;
    }
    if (row < a.M) qkv_epilogue<TN>(a, ni, row, v);
  }
}

// Persistent tile loop: a grid of at most one CTA per SM walks the output
// tiles t = blockIdx.x, blockIdx.x + gridDim.x, ...  Tiles are numbered in
// groups of kGroupN column tiles: inside a group the column tile varies
// fastest, then the row tile, so the ~gridDim.x tiles in flight share a few
// row blocks of A and kGroupN column blocks of W, both of which stay in L2.
// Six warps: warp 0 (one lane) streams A/W stages with TMA, warp 1 (one
// lane) issues the MMAs, warps 2-5 run the epilogue.  The accumulator is
// double-buffered in TMEM (2 x 256 columns), so the epilogue of tile i
// overlaps the MMAs of tile i + 1.
constexpr int kGroupN = 8;
constexpr int kEpiWarps = 4;
constexpr int kGemmThreads = 32 * (2 + kEpiWarps);
constexpr int kAccCols = 256;                 // columns per accumulator buffer
constexpr int kSmallPair = 72;                // gate (= up) rows of a small-M SwiGLU tile

struct TileGrid {
  int mt, nt;                                 // row / column tiles
  int ks, kbs;                                // K splits, K blocks per split
  __device__ __forceinline__ int count() const { return mt * nt * ks; }
  // work item t -> (row tile m, column tile n, K split z); the K split is
  // the slowest index, so concurrent CTAs share the A rows of one split
  __device__ __forceinline__ void at(int t, int& m, int& n, int& z) const {
    z = t / (mt * nt);
    t -= z * (mt * nt);
    const int per = kGroupN * mt;             // tiles per column group
    const int g = t / per, r = t - g * per;
    const int gw = min(kGroupN, nt - g * kGroupN);   // width of this group
    m = r / gw;
    n = g * kGroupN + (r - m * gw);
  }
};

// TN: tile columns (MMA N): 256 for TC_PLAIN / TC_SWIGLU, hd for TC_QKV.
template <int MODE, int TN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA,
               const __grid_constant__ CUtensorMap tmB, const TcArgs a,
               const TileGrid tg) {
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment of the swizzled tiles (shared-window address)
  const uint32_t raw = su32(smem_raw);
  uint8_t* base = smem_raw + ((1024 - (raw & 1023)) & 1023);
  uint8_t* sA = base;
  uint8_t* sB = base + STAGES * kStageA;
  __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ int s_fail, s_issued;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int OUTC = MODE == TC_SWIGLU ? TN / 2 : TN;   // output columns
  const int KB = a.K / BK;
  constexpr uint32_t kB = (uint32_t)TN * BK * 2;          // B bytes per stage
  volatile int* fail = &s_fail;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, kEpiWarps);
    }
    mbar_init(&mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
    s_fail = 0;
    s_issued = 0;
  }
  if (warp == 0) tmem_alloc(&tmem_base, 2 * kAccCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  pdl_wait();
  pdl_trigger();
  const int ntiles = tg.count();

  if (warp == 0) {
    // ---- TMA producer ----------------------------------------------------
    if (lane == 0) {
      int g = 0;                                // stage counter over all tiles
      for (int t = blockIdx.x; t < ntiles && !*fail; t += gridDim.x) {
        int mi, ni, z;
        tg.at(t, mi, ni, z);
        const int m0 = mi * BM, n0 = ni * OUTC;
        const int kb0 = z * tg.kbs, kb1 = min(KB, kb0 + tg.kbs);
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const int s = g % STAGES, use = g / STAGES;
          if (use > 0 && !mbar_wait(empty + s, (uint32_t)((use - 1) & 1))) {
            atomicOr(&s_fail, 1);
            break;
          }
          mbar_expect_tx(full + s, kStageA + kB);
          tma_load_2d(sA + s * kStageA, &tmA, kb * BK, m0, full + s);
          if (MODE == TC_QKV) {
            tma_load_2d(sB + s * kStageB, &tmB, kb * BK, ni * TN, full + s);
          } else {
            const int nb1 = MODE == TC_SWIGLU ? a.up_off + n0 : n0 + TN / 2;
            tma_load_2d(sB + s * kStageB, &tmB, kb * BK, n0, full + s);
            tma_load_2d(sB + s * kStageB + kB / 2, &tmB, kb * BK, nb1, full + s);
          }
          s_issued = g + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer --------------------------------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(BM, TN);
      int g = 0, i = 0;
      for (int t = blockIdx.x; t < ntiles && !*fail; t += gridDim.x, ++i) {
        const int buf = i & 1, ub = i >> 1;
        // the epilogue has drained this accumulator buffer (tile i - 2)
        if (ub > 0 && !mbar_wait(acc_empty + buf, (uint32_t)((ub - 1) & 1))) {
          atomicOr(&s_fail, 1);
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + buf * kAccCols;
        const int kb0 = (t / (tg.mt * tg.nt)) * tg.kbs;
        const int kb1 = min(KB, kb0 + tg.kbs);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
          const int s = g % STAGES, use = g / STAGES;
          if (!mbar_wait(full + s, (uint32_t)(use & 1))) {
            atomicOr(&s_fail, 1);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = su32(sA + s * kStageA), b0 = su32(sB + s * kStageB);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16(acc, smem_desc(a0 + kk * 32), smem_desc(b0 + kk * 32), idesc,
                      (kb - kb0 | kk) != 0);
          umma_commit(empty + s);                 // stage free once read
        }
        umma_commit(acc_full + buf);              // this tile's accumulator
        if (!ok) break;
      }
      // every MMA issued so far has completed once this arrives
      umma_commit(&mma_done);
    }
  } else {
    // ---- epilogue warps: TMEM -> registers -> global -------------------
    const int q = warp & 3;                       // TMEM lane quarter
    int i = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++i) {
      const int buf = i & 1, ub = i >> 1;
      const bool got = !*fail && mbar_wait(acc_full + buf, (uint32_t)(ub & 1));
      if (!got) {
        if (lane == 0) atomicOr(&s_fail, 1);
        break;
      }
      tc_fence_after();
      int mi, ni, z;
      tg.at(t, mi, ni, z);
      const int m0 = mi * BM, n0 = ni * OUTC;
      const int row = m0 + q * 32 + lane;
      const uint32_t trow = tmem + buf * kAccCols + ((uint32_t)(q * 32) << 16);
      epilogue_row<MODE, TN>(a, trow, row, n0, ni, z);
      // this warp's lanes are read: the buffer may take tile i + 2
      tc_fence_before();
      __syncwarp();
      if (lane == 0)
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(
                         su32(acc_empty + buf))
                     : "memory");
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the MMAs (and, after a failure, the copies) must be done before the
    // shared memory and TMEM are released
    if (!mbar_wait(&mma_done, 0)) atomicOr(&s_fail, 1);
    if (*fail) {
      atomicOr(a.err, ERRBIT_TIMEOUT);
      const int hi = s_issued, lo = hi > STAGES ? hi - STAGES : 0;
      for (int g = lo; g < hi; ++g)
        if (!mbar_wait(full + g % STAGES, (uint32_t)((g / STAGES) & 1))) break;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_free(tmem, 2 * kAccCols);
  }
}

// CTA-pair variant for many-row GEMMs (prefill): a cluster of two CTAs on
// one TPC computes a 256 x 256 output tile with tcgen05 cta_group::2 MMAs
// (M = 256, N = 256, K = 16).  Each CTA stages its own 128 rows of A and
// half of the tile's W rows (128: the first or second half of the column
// tile; SwiGLU: the gate rows in the even CTA, the up rows in the odd one),
// so a CTA moves 32 KB per 64-deep K block instead of 48 KB and the ring
// holds PSTAGES = 6 stages in the same shared memory.  Per K block each SM
// reads 16 KB of operands for 2 x 128 x 256 x 64 products, two thirds of
// what a one-CTA 128 x 256 tile reads: the single-CTA kernel is limited by
// the shared-memory bandwidth that the TMA fill and the MMA operand reads
// share.
//   both CTAs, warp 0 lane 0: TMA producer for its own halves; the copies
//       count on the even CTA's `full` barrier (the even producer arms it
//       with both CTAs' bytes), stages are released to both producers by
//       the MMA commit (multicast to both CTAs' `empty` barriers);
//   even CTA, warp 1 lane 0: MMA issuer (cta_group::2) into one of two
//       256-column accumulators of both CTAs' TMEM;
//   both CTAs, warps 2-5: epilogue of their own 128 rows (TMEM lanes), then
//       an arrival on the even CTA's `acc_empty` (8 arrivals per use).
// Every wait is bounded; a final cluster barrier keeps either CTA from
// leaving while the other may still address its shared memory or TMEM.
// Stage bytes per CTA (A rows + half the W rows) and ring depth for tile
// width TN (6 stages of 32 KB at TN = 256).
constexpr uint32_t pair_b_bytes(int TN) { return (uint32_t)(TN / 2) * BK * 2; }
constexpr uint32_t pair_stage_bytes(int TN) { return kStageA + pair_b_bytes(TN); }
constexpr int pair_stages(int TN) {
  return (int)(212992u / pair_stage_bytes(TN)) < 8 ? (int)(212992u / pair_stage_bytes(TN)) : 8;
}

template <int MODE, int TN>
__global__ void __launch_bounds__(kGemmThreads, 1)
gemm_tc_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                    const __grid_constant__ CUtensorMap tmB, const TcArgs a,
                    const TileGrid tg) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = su32(smem_raw);
  uint8_t* base = smem_raw + ((1024 - (raw & 1023)) & 1023);
  uint8_t* sA = base;
  constexpr int PSTAGES = pair_stages(TN);
  constexpr uint32_t kPairB = pair_b_bytes(TN), kPairStage = pair_stage_bytes(TN);
  uint8_t* sB = base + PSTAGES * kStageA;
  __shared__ __align__(8) uint64_t full[PSTAGES], empty[PSTAGES];
  __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_done;
  __shared__ uint32_t tmem_base;
  __shared__ int s_fail, s_issued;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();             // 0: MMA issuer
  constexpr int OUTC = MODE == TC_SWIGLU ? TN / 2 : TN;
  const int KB = a.K / BK;
  volatile int* fail = &s_fail;

  if (threadIdx.x == 0) {
    for (int i = 0; i < PSTAGES; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(acc_full + i, 1);
      mbar_init(acc_empty + i, 2 * kEpiWarps);
    }
    mbar_init(&mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
    s_fail = 0;
    s_issued = 0;
  }
  if (warp == 0) tmem_alloc_pair(&tmem_base, 2 * kAccCols);
  tc_fence_before();
  cluster_sync_all();             // both CTAs' barriers initialised, TMEM held
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  pdl_wait();
  pdl_trigger();
  const int ntiles = tg.count();
  const int c0 = blockIdx.x >> 1, nc = gridDim.x >> 1;   // cluster index, count
  const uint32_t full0 = cluster_addr(full, 0);          // the even CTA's
  const uint32_t acc_empty0 = cluster_addr(acc_empty, 0);

  if (warp == 0) {
    // ---- TMA producer (both CTAs) -----------------------------------------
    if (lane == 0) {
      int g = 0;
      for (int t = c0; t < ntiles && !*fail; t += nc) {
        int mi, ni, z;
        tg.at(t, mi, ni, z);
        const int m0 = mi * 2 * BM + (int)rank * BM;
        const int nb = MODE == TC_SWIGLU ? (rank ? a.up_off : 0) + ni * OUTC
                                         : ni * TN + (int)rank * (TN / 2);
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % PSTAGES, use = g / PSTAGES;
          if (use > 0 && !mbar_wait(empty + s, (uint32_t)((use - 1) & 1))) {
            atomicOr(&s_fail, 1);
            break;
          }
          if (rank == 0) mbar_expect_tx(full + s, 2 * kPairStage);
          tma_load_2d_pair(sA + s * kStageA, &tmA, kb * BK, m0, full0 + 8 * s);
          tma_load_2d_pair(sB + s * kPairB, &tmB, kb * BK, nb, full0 + 8 * s);
          s_issued = g + 1;
        }
      }
    }
  } else if (warp == 1) {
    // ---- MMA issuer (even CTA) --------------------------------------------
    if (lane == 0 && rank == 0) {
      constexpr uint32_t idesc = idesc_bf16(2 * BM, TN);
      int g = 0, i = 0;
      for (int t = c0; t < ntiles && !*fail; t += nc, ++i) {
        const int buf = i & 1, ub = i >> 1;
        // both CTAs' epilogues have drained this buffer (tile i - 2)
        if (ub > 0 && !mbar_wait_cluster(acc_empty + buf, (uint32_t)((ub - 1) & 1))) {
          atomicOr(&s_fail, 1);
          break;
        }
        tc_fence_after();
        const uint32_t acc = tmem + buf * kAccCols;
        bool ok = true;
        for (int kb = 0; kb < KB; ++kb, ++g) {
          const int s = g % PSTAGES, use = g / PSTAGES;
          if (!mbar_wait(full + s, (uint32_t)(use & 1))) {
            atomicOr(&s_fail, 1);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = su32(sA + s * kStageA), b0 = su32(sB + s * kPairB);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16_pair(acc, smem_desc(a0 + kk * 32), smem_desc(b0 + kk * 32),
                           idesc, (kb | kk) != 0);
          umma_commit_pair(empty + s);           // both CTAs' stage s is free
        }
        umma_commit_pair(acc_full + buf);
        if (!ok) break;
      }
      umma_commit_pair(&mma_done);
    }
  } else {
    // ---- epilogue warps (both CTAs): own 128 rows --------------------------
    const int q = warp & 3;
    int i = 0;
    for (int t = c0; t < ntiles; t += nc, ++i) {
      const int buf = i & 1, ub = i >> 1;
      const bool got = !*fail && mbar_wait(acc_full + buf, (uint32_t)(ub & 1));
      if (!got) {
        if (lane == 0) atomicOr(&s_fail, 1);
        break;
      }
      tc_fence_after();
      int mi, ni, z;
      tg.at(t, mi, ni, z);
      const int row = mi * 2 * BM + (int)rank * BM + q * 32 + lane;
      const uint32_t trow = tmem + buf * kAccCols + ((uint32_t)(q * 32) << 16);
      epilogue_row<MODE, TN>(a, trow, row, ni * OUTC, ni, 0);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc_empty0 + 8 * buf);
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // the pair's MMAs read this CTA's shared memory and write its TMEM: all
    // of them must be done before either is released (the commit reaches
    // both CTAs)
    if (!mbar_wait(&mma_done, 0)) atomicOr(&s_fail, 1);
    if (*fail) {
      atomicOr(a.err, ERRBIT_TIMEOUT);
      if (rank == 0) {
        const int hi = s_issued, lo = hi > PSTAGES ? hi - PSTAGES : 0;
        for (int g = lo; g < hi; ++g)
          if (!mbar_wait(full + g % PSTAGES, (uint32_t)((g / PSTAGES) & 1), kSpin / 16))
            break;
      }
    }
  }
  tc_fence_before();
  cluster_sync_all();
  if (warp == 0) {
    tc_fence_after();
    tmem_free_pair(tmem, 2 * kAccCols);
  }
}

// ---------------------------------------------------------------- host ----
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 tensor map over rows x cols (cols contiguous, row stride ld
// elements), box `brows` rows x 64 columns, 128-byte swizzle, zero fill.
bool make_map(CUtensorMap* m, const void* ptr, long rows, long cols, long ld,
              int brows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {BK, (cuuint32_t)brows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool make_map_2d(CUtensorMap* m, const void* ptr, long rows, long cols,
                 long ld, int box_cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn || (box_cols != 32 && box_cols != 64)) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_kv_tile_map(CUtensorMap* m, const void* ptr, long rows, int hd) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)hd, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)hd * 2};
  cuuint32_t box[2] = {32, (cuuint32_t)kv_tile_rows()};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// Tensor maps of weights are built once per (pointer, shape, box).
std::mutex g_map_mu;
std::map<std::tuple<const void*, long, long, int>, CUtensorMap> g_maps;

bool weight_map(CUtensorMap* m, const void* ptr, long rows, long cols,
                int brows) {
  std::lock_guard<std::mutex> lock(g_map_mu);
  auto key = std::make_tuple(ptr, rows, cols, brows);
  auto it = g_maps.find(key);
  if (it != g_maps.end()) {
    *m = it->second;
    return true;
  }
  if (!make_map(m, ptr, rows, cols, cols, brows)) return false;
  g_maps[key] = *m;
  return true;
}

// CTA-pair tiles for many-row GEMMs (DORY_PAIR_GEMM=0 keeps one CTA per
// 128 x 256 tile everywhere).
bool pair_gemm_enabled() {
  static const bool on = [] {
    const char* e = getenv("DORY_PAIR_GEMM");
    return !(e && e[0] == '0');
  }();
  return on;
}

int* g_err_ptr = nullptr;

size_t tc_smem() { return (size_t)STAGES * (kStageA + kStageB) + 1024; }

int num_sms() {
  static int n = [] {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 1;
  }();
  return n;
}

// tiles: row tiles x column tiles of the output; one persistent CTA per SM
// at most
template <int MODE, int TN>
bool launch_tc(const CUtensorMap& ma, const CUtensorMap& mb, const TcArgs& a,
               int mt, int nt, cudaStream_t st, int ks = 1) {
  static bool configured = false;
  if (!configured) {
    cudaFuncSetAttribute(gemm_tc_kernel<MODE, TN>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)tc_smem());
    configured = true;
  }
  const int KB = a.K / BK;
  const int kbs = (KB + ks - 1) / ks;
  const TileGrid tg{mt, nt, (KB + kbs - 1) / kbs, kbs};
  const int tiles = mt * nt * tg.ks;
  const int grid = tiles < num_sms() ? tiles : num_sms();
  return launch_k(gemm_tc_kernel<MODE, TN>, dim3(grid), dim3(kGemmThreads),
                  tc_smem(), st, ma, mb, a, tg) == cudaSuccess;
}

template <int TN>
size_t tc_pair_smem() {
  return (size_t)pair_stages(TN) * pair_stage_bytes(TN) + 1024;
}

// Clusters of two co-resident at once (one CTA per SM), at most.
template <int MODE, int TN>
int pair_clusters() {
  static int n = [] {
    cudaFuncSetAttribute(gemm_tc_pair_kernel<MODE, TN>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)tc_pair_smem<TN>());
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(num_sms() >= 2 ? num_sms() & ~1 : 2);   // whole pairs
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = tc_pair_smem<TN>();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int v = 0;
    if (cudaOccupancyMaxActiveClusters(&v, gemm_tc_pair_kernel<MODE, TN>, &cfg) !=
            cudaSuccess || v < 1) {
      cudaGetLastError();
      v = num_sms() / 2;
    }
    return v;
  }();
  return n;
}

// Pair tiles: mt2 row tiles of 256 rows x nt column tiles of TN.
template <int MODE, int TN>
bool launch_tc_pair(const CUtensorMap& ma, const CUtensorMap& mb,
                    const TcArgs& a, int mt2, int nt, cudaStream_t st) {
  const int clusters = pair_clusters<MODE, TN>();
  const int KB = a.K / BK;
  const TileGrid tg{mt2, nt, 1, KB};
  const int tiles = mt2 * nt;
  const int grid = 2 * (tiles < clusters ? tiles : clusters);
  return launch_k_cluster(gemm_tc_pair_kernel<MODE, TN>, dim3(grid),
                          dim3(kGemmThreads), tc_pair_smem<TN>(), st, 2, ma, mb,
                          a, tg) == cudaSuccess;
}

TcArgs base_args(int M, int N, int K) {
  TcArgs a{};
  a.M = M;
  a.N = N;
  a.K = K;
  a.err = g_err_ptr;
  return a;
}

}  // namespace

void set_tc_error_word(int* err) { g_err_ptr = err; }

// C[M, N] = A[M, K] W[N, K]^T (f32, optional column scale) on tcgen05.
// With max_splits > 1 and fewer output tiles than SMs, K is split so that
// about one work item runs per SM: split z writes its f32 partial to
// C + z * slab and the reader sums the partials.  Returns the split count.
int launch_gemm_bf16(const bf16* A, int lda, const bf16* W, float* C, int ldc,
                     int M, int N, int K, const float* col_scale,
                     cudaStream_t st, int max_splits, long slab,
                     const float* out_scale) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K, lda, BM) || !weight_map(&mb, W, N, K, 128)) {
    note_host_failure("gemm: tensor map");
    return 1;
  }
  TcArgs a = base_args(M, N, K);
  a.C = C;
  a.ldc = ldc;
  a.slab = slab;
  a.col_scale = col_scale;
  a.out_scale = out_scale;
  const int mt = (M + BM - 1) / BM, nt = (N + BN - 1) / BN;
  const int ks = gemm_split_count(M, N, K, col_scale ? 1 : max_splits);
  if (ks == 1 && mt > 1 && pair_gemm_enabled())
    launch_tc_pair<TC_PLAIN, BN>(ma, mb, a, (M + 2 * BM - 1) / (2 * BM), nt, st);
  else
    launch_tc<TC_PLAIN, BN>(ma, mb, a, mt, nt, st, ks);
  return ks;
}

int gemm_split_count(int M, int N, int K, int max_splits) {
  const int mt = (M + BM - 1) / BM, nt = (N + BN - 1) / BN;
  const int KB = K / BK;
  int ks = 1;
  if (max_splits > 1 && mt * nt < num_sms()) {
    // at least 2 K blocks per split keep the stage ring busy
    ks = std::min(std::min(max_splits, num_sms() / (mt * nt)), KB / 2);
    if (ks < 1) ks = 1;
    const int kbs = (KB + ks - 1) / ks;
    ks = (KB + kbs - 1) / kbs;                  // no empty split
  }
  return ks;
}

// m[M, F] = silu(A W_g^T) * (A W_u^T) (bf16) with W = [W_g; W_u] of 2F rows.
void launch_gemm_swiglu(const bf16* A, int lda, const bf16* W, bf16* m,
                        int ldm, int M, int F, int K, cudaStream_t st,
                        const float* out_scale) {
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, M, K, lda, BM) || !weight_map(&mb, W, 2L * F, K, 128)) {
    note_host_failure("gemm: tensor map");
    return;
  }
  TcArgs a = base_args(M, F, K);
  a.out_scale = out_scale;
  a.up_off = F;
  a.Cb = m;
  a.ldc = ldm;
  const int mt = (M + BM - 1) / BM;
  if (mt == 1 && (F + kSmallPair - 1) / kSmallPair <= num_sms()) {
    // one row tile (decode batches): 72 gate + 72 up rows per tile, so that
    // the F / 72 tiles (143 for F = 10240) give every SM one tile
    CUtensorMap mb2;
    if (!weight_map(&mb2, W, 2L * F, K, kSmallPair)) {
      note_host_failure("gemm: tensor map");
      return;
    }
    launch_tc<TC_SWIGLU, 2 * kSmallPair>(ma, mb2, a, mt,
                                         (F + kSmallPair - 1) / kSmallPair, st);
    return;
  }
  if (pair_gemm_enabled())
    launch_tc_pair<TC_SWIGLU, BN>(ma, mb, a, (M + 2 * BM - 1) / (2 * BM),
                                  (F + BN / 2 - 1) / (BN / 2), st);
  else
    launch_tc<TC_SWIGLU, BN>(ma, mb, a, mt, (F + BN / 2 - 1) / (BN / 2), st);
}

// Fused q/k/v/gate projection with the RoPE / QK-norm / KV-write epilogue.
void launch_gemm_qkv(const bf16* A, int lda, const bf16* W, const QkvGemmArgs& q,
                     cudaStream_t st, const float* out_scale) {
  const int hd = q.dm.hd;
  const int rows = q.dm.rows_qkvg;
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, q.M, q.dm.d, lda, BM) ||
      !weight_map(&mb, W, rows, q.dm.d, hd)) {
    note_host_failure("gemm: tensor map");
    return;
  }
  TcArgs a = base_args(q.M, rows, q.dm.d);
  a.out_scale = out_scale;
  a.T = q.T;
  a.Hq = q.dm.Hq;
  a.Hkv = q.dm.Hkv;
  a.qdim = q.dm.qdim;
  a.kvdim = q.dm.kvdim;
  a.s_q = q.s_q;
  a.s_k = q.s_k;
  a.rope = q.rope;
  a.q_scale = q.q_scale;
  a.kv = q.kv;
  a.g = q.g;
  a.q_out = q.q_out;
  a.gate_out = q.gate_out;
  a.row_loops = q.row_loops;
  a.loop_t = q.loop_t;
  const int mt = (q.M + BM - 1) / BM, nt = rows / hd;
  switch (hd) {
    case 64: launch_tc<TC_QKV, 64>(ma, mb, a, mt, nt, st); break;
    case 128: launch_tc<TC_QKV, 128>(ma, mb, a, mt, nt, st); break;
    default: launch_tc<TC_QKV, 160>(ma, mb, a, mt, nt, st); break;
  }
}

}  // namespace dory
