// Decode attention (one query token per sequence) over the paged / ring KV
// cache: one thread-block cluster per (sequence, KV head) splits the key
// range, TMA-fed stages feed the warp-level tensor cores, and the cluster
// merges its splits through distributed shared memory.
//
// Visible keys for the query at position p: j <= p, and for sliding-window
// layers also j > p - W (W = 1024 for Dory; the paper summary, 技术新颖性:
// 3:1 sliding-window to full attention).  Query head h reads KV head h / G,
// G = Hq / Hkv.  Scores are in exp2 units: q arrives pre-multiplied by
// sqrt(head_dim) * log2(e), so exp2(q.k - m) is the softmax numerator.  The
// gate sigmoid(g) multiplies the head outputs; the L2 norm of the gated
// concatenation that precedes W_o (paperlayer §2) is folded into the
// normalised update that follows W_o (N(W N(a)) = N(W a)).
//
// Keys go in tiles of 32 positions aligned to multiples of 32, so a tile lies
// inside one 64-token page (full layers) or one run of ring slots (sliding-
// window layers, whose ring capacity is a multiple of 32).  A tile's K and V
// rows arrive by 2-D TMA loads (box 32 keys x 32 dims with the 64-byte
// swizzle, head_dim / 32 boxes per matrix) into a ring of three stages.
//
// grid (C, Hkv, B), clusters of C blocks along x (C = 16, or 8 where 16-block
// clusters do not fit); block rank r takes tiles [t0 + r c, t0 + (r+1) c) of
// the visible range, c = ceil(tiles / C).  Block of 96 threads:
//   warp 0, lane 0  loads the block's tiles through the stage ring; the first
//                   stages are issued before the dependency wait (positions
//                   < p were written by finished calls; row p is replaced in
//                   shared memory);
//   warps 1-2       (a) every block forms the vectors it reads from the
//                   QKVG partials (rotate-half RoPE, per-head L2 norm,
//                   scales; k and v rounded to BF16): q_0 .. q_{G-1}, and in
//                   the block holding position p also k and v (forming them
//                   locally, all loads in one L2 round trip, is quicker than
//                   a cluster barrier and a copy from owner blocks);
//                   (b) the block holding position p stores k, v in the cache;
//                   (c) per stage warp c takes keys 16c..16c+15: S^T = K Q^T
//                   on m16n8k16 (K rows as A, the heads as the 8 columns),
//                   masked online softmax per head (lane 4g + t owns heads 2t,
//                   2t+1), P^T by an in-register transpose, O^T += V^T P^T
//                   (V rows through ldmatrix.trans);
//                   (d) the block's (m, l, O) per head goes to shared memory;
//                   after a cluster barrier block r merges output slice r of
//                   the G x head_dim outputs over the C blocks (exact
//                   max-rescaled sums in rank order), applies sigmoid(gate)
//                   and writes bf16; a last cluster barrier keeps every
//                   block's shared memory alive until its readers are done.
// Every mbarrier wait is bounded: a timeout sets ERRBIT_TIMEOUT and the block
// carries on through the cluster barriers (which every thread reaches on
// every path) and waits (bounded) for its own copies before exiting.
#include "async_copy.cuh"
#include "common.cuh"
#include "warp_mma.cuh"

namespace dory {

namespace {

constexpr int DTK = 32;                       // keys per tile (one stage)
constexpr int kStages = 3;
constexpr int kCons = 2;                      // consumer warps
constexpr int kDecThreads = 32 * (1 + kCons);
constexpr int kPanelBytes = DTK * 64;         // one box: 32 keys x 32 dims
constexpr int kMaxCluster = 16;

// First row of tile t of (b, kvh) in the 2-D [rows][head_dim] view of the
// cache: ring slots [B][Hkv][cap] or pages [n_pages][Hkv][kPage].
__device__ __forceinline__ int tile_row(const KVSlot& kv, const CacheGeo& g,
                                        int Hkv, int b, int kvh, int t) {
  const int j = t * DTK;
  if (kv.ring) return (b * Hkv + kvh) * kv.cap + j % kv.cap;
  const int page = g.block_table[b * g.pages_per_seq + j / kPage];
  return (page * Hkv + kvh) * kPage + j % kPage;
}

// Byte offset of (row r, 16-byte chunk c) in a panel stored with the 64-byte
// swizzle (chunk index XOR bits 1-2 of the row; panels are 512-byte aligned).
__device__ __forceinline__ uint32_t swz64(int r, int c) {
  return (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ void cons_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * kCons) : "memory");
}

// ---- thread-block cluster: barrier and distributed shared memory ----------
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in block `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(const void* p, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;"
               : "=r"(r)
               : "r"(su32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_peer(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ float4 ld_peer4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// One warp forms up to NW vectors v of (q_0 .. q_{G-1}, k, v) of KV head kvh
// (vs[j] < 0: none) from the split-K partials of the fused QKVG output: q and
// k get rotate-half RoPE (rope: [hd/2] cos, sin of this position), the L2
// norm over the head and the per-dim scale (q also q_scale); k and v are
// rounded to BF16, the precision the cache holds.  Every load of every
// vector is issued before the first use (one L2 round trip).
template <int HD, int G, int NW>
__device__ __forceinline__ void form_vectors(const DecAttnArgs& a,
                                             const float* src, size_t pstride,
                                             int kvh, const int (&vs)[NW],
                                             float* vec_s) {
  constexpr int HALF = HD / 2;
  constexpr int NPR = (HALF + 31) / 32;       // rotation pairs per lane
  const Dims& dm = a.dm;
  const int lane = threadIdx.x & 31;
  float x1[NW][NPR], x2[NW][NPR], cs[NPR], sn[NPR], sc1[NW][NPR], sc2[NW][NPR];
#pragma unroll
  for (int j = 0; j < NPR; ++j) {
    const int i = lane + 32 * j;
    cs[j] = i < HALF ? a.rope[2 * i] : 0.f;
    sn[j] = i < HALF ? a.rope[2 * i + 1] : 0.f;
  }
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int v = vs[w];
    const bool is_q = v < G, is_v = v == G + 1;
    const float* scale = is_q ? a.s_q + (kvh * G + v) * HD : a.s_k + kvh * HD;
#pragma unroll
    for (int j = 0; j < NPR; ++j) {
      const int i = lane + 32 * j;
      const bool in = v >= 0 && i < HALF && !is_v;
      x1[w][j] = x2[w][j] = 0.f;
      sc1[w][j] = in ? scale[i] : 0.f;
      sc2[w][j] = in ? scale[i + HALF] : 0.f;
    }
  }
  for (int s = 0; s < a.S; ++s) {
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const int v = vs[w];
      if (v < 0) continue;
      const bool is_q = v < G, is_v = v == G + 1;
      const int col0 = is_q ? (kvh * G + v) * HD
                     : !is_v ? dm.qdim + kvh * HD : dm.qdim + dm.kvdim + kvh * HD;
      const float* sp = src + s * pstride + col0;
#pragma unroll
      for (int j = 0; j < NPR; ++j) {
        const int i = lane + 32 * j;
        if (i < HALF) {
          x1[w][j] += sp[i];
          x2[w][j] += sp[i + HALF];
        }
      }
    }
  }
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    const int v = vs[w];
    if (v < 0) continue;
    const bool is_q = v < G, is_v = v == G + 1;
    float* dst = vec_s + v * HD;
    if (is_v) {
#pragma unroll
      for (int j = 0; j < NPR; ++j) {
        const int i = lane + 32 * j;
        if (i < HALF) {
          dst[i] = __bfloat162float(__float2bfloat16_rn(x1[w][j]));
          dst[i + HALF] = __bfloat162float(__float2bfloat16_rn(x2[w][j]));
        }
      }
      continue;
    }
    float r1[NPR], r2[NPR], ss = 0.f;
#pragma unroll
    for (int j = 0; j < NPR; ++j) {
      r1[j] = x1[w][j] * cs[j] - x2[w][j] * sn[j];
      r2[j] = x2[w][j] * cs[j] + x1[w][j] * sn[j];
      ss += r1[j] * r1[j] + r2[j] * r2[j];
    }
    const float inv = 1.f / fmaxf(sqrtf(warp_sum(ss)), 1e-12f);
    const float extra = is_q ? a.q_scale : 1.f;
#pragma unroll
    for (int j = 0; j < NPR; ++j) {
      const int i = lane + 32 * j;
      if (i < HALF) {
        float u = r1[j] * inv * sc1[w][j] * extra;
        float z = r2[j] * inv * sc2[w][j] * extra;
        if (!is_q) {
          u = __bfloat162float(__float2bfloat16_rn(u));
          z = __bfloat162float(__float2bfloat16_rn(z));
        }
        dst[i] = u;
        dst[i + HALF] = z;
      }
    }
  }
}

template <int HD, int G>
__global__ void __launch_bounds__(kDecThreads)
attn_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV,
                   const DecAttnArgs a) {
  static_assert(HD % 32 == 0 && G >= 1 && G <= 8, "head_dim % 32, G <= 8");
  constexpr int NP = HD / 32;                 // boxes (panels) per K or V tile
  constexpr int SK = NP * kPanelBytes;        // bytes of K (or V) per stage
  constexpr int KS = HD / 16;                 // 16-dim blocks of a head
  constexpr int CT = 32 * kCons;              // consumer threads
  constexpr int NV = G + 2;                   // formed vectors: q heads, k, v
  constexpr int NOUT = (G * HD + 8 * CT - 1) / (8 * CT);   // outputs / thread
  extern __shared__ uint8_t smraw[];
  uint8_t* tiles = smraw + ((1024 - (su32(smraw) & 1023)) & 1023);
  float* vec_s = reinterpret_cast<float*>(tiles + kStages * 2 * SK);  // [NV][HD]
  float* q_s = vec_s;                         // [G][HD]
  float* kn_s = vec_s + G * HD;               // [HD] new k
  float* vn_s = kn_s + HD;                    // [HD] new v
  float* part = vn_s + HD;                    // block partial: m[G] l[G] O[G][HD]
  float* comb = part + G * (HD + 2);          // warp states [kCons][G][HD + 2]
  __shared__ __align__(8) uint64_t full[kStages], empty[kStages];
  __shared__ int s_fail, s_issued;
  volatile int* fail = &s_fail;

  const Dims& dm = a.dm;
  const int C = gridDim.x;                    // blocks per cluster (= grid x)
  const int b = blockIdx.z, kvh = blockIdx.y, rank = blockIdx.x;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int p = *a.g.n_ctx;
  if (p >= a.g.max_ctx) {                     // uniform over the grid
    pdl_wait();
    if (rank == 0 && kvh == 0 && tid == 0) atomicOr(a.err, ERRBIT_BOUNDS);
    return;
  }
  const int lo = a.window ? max(0, p - a.window + 1) : 0;
  const int t0 = lo / DTK, nt = p / DTK - t0 + 1;
  const int chunk = (nt + C - 1) / C;
  const int tb = t0 + rank * chunk;           // first tile of this block
  const int ntile = max(0, min(t0 + nt, tb + chunk) - tb);
  const bool has_p = ntile > 0 && tb + ntile == t0 + nt;   // tile of p

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, kCons);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    s_fail = 0;
    s_issued = 0;
  }
  __syncthreads();

  if (w == 0) {
    // ---- producer ----------------------------------------------------------
    const CUtensorMap* mk = &tmK;
    const CUtensorMap* mv = &tmV;
    auto issue = [&](int i) {
      const int s = i % kStages;
      const int row = tile_row(a.kv, a.g, dm.Hkv, b, kvh, tb + i);
      uint8_t* kt = tiles + s * 2 * SK;
      mbar_expect_tx(full + s, 2 * SK);
#pragma unroll
      for (int pp = 0; pp < NP; ++pp) {
        tma_load_2d(kt + pp * kPanelBytes, mk, pp * 32, row, full + s);
        tma_load_2d(kt + SK + pp * kPanelBytes, mv, pp * 32, row, full + s);
      }
      s_issued = i + 1;
    };
    if (lane == 0)
      for (int i = 0; i < min(kStages, ntile); ++i) issue(i);
    __syncwarp();
    pdl_wait();
    pdl_trigger();
    if (lane != 0) {
      // weights of the next projections into L2, once the predecessor's
      // weight stream has ended
      const void* pp[kMaxL2Ranges];
      long pb[kMaxL2Ranges];
#pragma unroll
      for (int r = 0; r < kMaxL2Ranges; ++r) {
        pp[r] = a.l2pf[r].p;
        pb[r] = a.l2pf[r].bytes;
      }
      const int parts = C * dm.Hkv * a.B;
      const int part = rank + C * (kvh + dm.Hkv * b);
      l2_prefetch_share<kMaxL2Ranges>(pp, pb, part, parts, lane - 1, 31);
    }
    if (lane == 0) {
      for (int i = kStages; i < ntile && !*fail; ++i) {
        // the consumers have released this stage's previous tile
        if (!mbar_wait(empty + i % kStages, (uint32_t)((i / kStages - 1) & 1))) {
          atomicOr(&s_fail, 1);
          break;
        }
        issue(i);
      }
    }
    __syncwarp();
    cluster_arrive();                         // (2)
    cluster_wait();
    cluster_arrive();                         // (3)
    cluster_wait();
  } else {
    // ---- consumers ---------------------------------------------------------
    pdl_wait();
    pdl_trigger();
    const int cw = w - 1, ct = tid - 32;
    const float* src = a.qkvg + (size_t)b * dm.rows_qkvg;
    const size_t pstride = (size_t)a.B * dm.rows_qkvg;

    // gate of this block's output slice [o0, o1), summed over the partials
    const int per = (G * HD + C - 1) / C;     // outputs merged per block
    const int o0 = rank * per, o1 = min(G * HD, o0 + per);
    float gate[NOUT];
#pragma unroll
    for (int k = 0; k < NOUT; ++k) {
      gate[k] = 0.f;
      const int idx = o0 + ct + k * CT;
      if (idx < o1)
        for (int s3 = 0; s3 < a.S; ++s3)
          gate[k] += src[s3 * pstride + dm.qdim + 2 * dm.kvdim + kvh * G * HD + idx];
    }

    // (a) every block forms the vectors it reads itself: the G query heads,
    // and where p's tile is, the new k and v (warp cw takes vectors cw,
    // cw + 2, ...); no cluster exchange is needed before the tiles
    {
      constexpr int NW = (NV + kCons - 1) / kCons;
      int vs[NW];
#pragma unroll
      for (int j = 0; j < NW; ++j) {
        const int v = cw + kCons * j;
        vs[j] = (v < G || (v < NV && has_p)) ? v : -1;
      }
      form_vectors<HD, G, NW>(a, src, pstride, kvh, vs, vec_s);
    }
    cons_sync();

    // (b) the block holding position p stores the new entry (not for a row
    // that sits out this loop)
    if (has_p && row_writes_kv(a.row_loops, b, a.loop_t)) {
      const size_t off = kv_index(a.kv, a.g, dm.Hkv, HD, b, kvh, p);
      for (int c = ct; c < HD; c += CT) {
        a.kv.K[off + c] = __float2bfloat16_rn(kn_s[c]);
        a.kv.V[off + c] = __float2bfloat16_rn(vn_s[c]);
      }
    }

    // (c) tiles.  Q^T as the B operand: lane (g, t) holds q[g][16k + 2t..]
    // and q[g][16k + 2t + 8..] of k-step k; heads g >= G are zero.
    const int g = lane >> 2, t = lane & 3;
    uint32_t qf[KS][2];
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      qf[ks][0] = qf[ks][1] = 0u;
      if (g < G) {
        const float* qr = q_s + g * HD + ks * 16 + 2 * t;
        qf[ks][0] = pack_bf16(qr[0], qr[1]);
        qf[ks][1] = pack_bf16(qr[8], qr[9]);
      }
    }
    const int kb = 16 * cw;                   // this warp's keys in a tile
    // ldmatrix row / chunk of this lane: K rows as A (x4 = keys 0-7 / 8-15 x
    // dims 0-7 / 8-15 of the k-step), V rows transposed (keys 0-7 / 8-15 x
    // dims 0-7 / 8-15 of the 16-dim block)
    const int rk = kb + (lane & 7) + 8 * ((lane >> 3) & 1), ck = lane >> 4;
    const int rv = kb + (lane & 7) + 8 * (lane >> 4), cv = (lane >> 3) & 1;
    float m2[2] = {-INFINITY, -INFINITY}, l2[2] = {0.f, 0.f};
    float o[KS][4];
#pragma unroll
    for (int d = 0; d < KS; ++d) o[d][0] = o[d][1] = o[d][2] = o[d][3] = 0.f;

    for (int i = 0; i < ntile; ++i) {
      const int s = i % kStages;
      if (!mbar_wait_warp(full + s, (uint32_t)((i / kStages) & 1))) {
        atomicOr(&s_fail, 1);
        break;
      }
      uint8_t* kt = tiles + s * 2 * SK;
      uint8_t* vt = kt + SK;
      const uint32_t ka = su32(kt), va = ka + SK;
      const int j0 = (tb + i) * DTK, jw = j0 + kb;
      bool touched = false;                   // generic writes to the stage
      if (p >= jw && p < jw + 16) {
        // the current token's row: the cache row may not hold it yet
        const int r = p - j0;
        for (int c = lane; c < HD / 8; c += 32) {
          uint4 kq, vq;
          kq.x = pack_bf16(kn_s[8 * c + 0], kn_s[8 * c + 1]);
          kq.y = pack_bf16(kn_s[8 * c + 2], kn_s[8 * c + 3]);
          kq.z = pack_bf16(kn_s[8 * c + 4], kn_s[8 * c + 5]);
          kq.w = pack_bf16(kn_s[8 * c + 6], kn_s[8 * c + 7]);
          vq.x = pack_bf16(vn_s[8 * c + 0], vn_s[8 * c + 1]);
          vq.y = pack_bf16(vn_s[8 * c + 2], vn_s[8 * c + 3]);
          vq.z = pack_bf16(vn_s[8 * c + 4], vn_s[8 * c + 5]);
          vq.w = pack_bf16(vn_s[8 * c + 6], vn_s[8 * c + 7]);
          const uint32_t off = (c >> 2) * kPanelBytes + swz64(r, c & 3);
          *reinterpret_cast<uint4*>(kt + off) = kq;
          *reinterpret_cast<uint4*>(vt + off) = vq;
        }
        touched = true;
      }
      if (jw < lo || jw + 15 > p) {
        // keys outside [lo, p] get probability 0; zero their V rows so that
        // whatever those cache rows hold cannot turn 0 * v into NaN
        for (int e = lane; e < 16 * (HD / 8); e += 32) {
          const int rr = e / (HD / 8), c = e - rr * (HD / 8);
          const int j = jw + rr;
          if (j < lo || j > p)
            *reinterpret_cast<uint4*>(vt + (c >> 2) * kPanelBytes +
                                      swz64(kb + rr, c & 3)) = make_uint4(0, 0, 0, 0);
        }
        touched = true;
      }
      __syncwarp();

      // S^T (16 keys x 8 heads) = K Q^T, two accumulators for ILP
      float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        uint32_t af[4];
        ldsm_x4(ka + (ks >> 1) * kPanelBytes + swz64(rk, 2 * (ks & 1) + ck), af[0],
                af[1], af[2], af[3]);
        if (ks & 1) mma16816(sb, af, qf[ks][0], qf[ks][1]);
        else mma16816(sa, af, qf[ks][0], qf[ks][1]);
      }
      // c0, c1: key jw + g, heads 2t, 2t + 1; c2, c3: key jw + g + 8
      const int ja = jw + g, jb = ja + 8;
      const bool oka = ja >= lo && ja <= p, okb = jb >= lo && jb <= p;
      float sc[4] = {oka ? sa[0] + sb[0] : -INFINITY, oka ? sa[1] + sb[1] : -INFINITY,
                     okb ? sa[2] + sb[2] : -INFINITY, okb ? sa[3] + sb[3] : -INFINITY};
      float mx[2] = {fmaxf(sc[0], sc[2]), fmaxf(sc[1], sc[3])};
#pragma unroll
      for (int sh = 4; sh < 32; sh <<= 1) {
        mx[0] = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], sh));
        mx[1] = fmaxf(mx[1], __shfl_xor_sync(0xffffffffu, mx[1], sh));
      }
      float corr[2], sum[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float mn = fmaxf(m2[h], mx[h]);
        const bool none = mn == -INFINITY;
        corr[h] = none ? 1.f : exp2f(m2[h] - mn);
        sc[h] = none ? 0.f : exp2f(sc[h] - mn);
        sc[h + 2] = none ? 0.f : exp2f(sc[h + 2] - mn);
        sum[h] = sc[h] + sc[h + 2];
        m2[h] = mn;
      }
#pragma unroll
      for (int sh = 4; sh < 32; sh <<= 1) {
        sum[0] += __shfl_xor_sync(0xffffffffu, sum[0], sh);
        sum[1] += __shfl_xor_sync(0xffffffffu, sum[1], sh);
      }
      l2[0] = l2[0] * corr[0] + sum[0];
      l2[1] = l2[1] * corr[1] + sum[1];
      // P^T as the B operand (keys x heads): transpose the key x head blocks
      const uint32_t pb0 = movmatrix_t(pack_bf16(sc[0], sc[1]));
      const uint32_t pb1 = movmatrix_t(pack_bf16(sc[2], sc[3]));
      // O^T (dims x heads) += V^T P^T
#pragma unroll
      for (int d = 0; d < KS; ++d) {
        o[d][0] *= corr[0];
        o[d][1] *= corr[1];
        o[d][2] *= corr[0];
        o[d][3] *= corr[1];
        uint32_t af[4];
        ldsm_x4_t(va + (d >> 1) * kPanelBytes + swz64(rv, 2 * (d & 1) + cv), af[0],
                  af[1], af[2], af[3]);
        mma16816(o[d], af, pb0, pb1);
      }
      // release the stage (generic writes ordered before the next TMA fill)
      if (touched) fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(empty + s);
    }

    // (d) the block's partial: the two warps' states combined
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int head = 2 * t + h;
      if (head < G) {
        float* ws = comb + (cw * G + head) * (HD + 2);
        if (g == 0) {
          ws[0] = m2[h];
          ws[1] = l2[h];
        }
#pragma unroll
        for (int d = 0; d < KS; ++d) {
          ws[2 + 16 * d + g] = o[d][h];
          ws[2 + 16 * d + g + 8] = o[d][h + 2];
        }
      }
    }
    cons_sync();
    for (int idx = ct; idx < G * (HD + 2); idx += CT) {
      const int gg = idx / (HD + 2), c = idx - gg * (HD + 2);
      float M = -INFINITY;
#pragma unroll
      for (int w2 = 0; w2 < kCons; ++w2) M = fmaxf(M, comb[(w2 * G + gg) * (HD + 2)]);
      float acc = M;
      if (c > 0) {
        acc = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kCons; ++w2) {
          const float* cs = comb + (w2 * G + gg) * (HD + 2);
          const float f = cs[0] == -INFINITY ? 0.f : exp2f(cs[0] - M);
          acc = fmaf(f, cs[c], acc);
        }
      }
      // part: m[G], l[G], then O[G][HD]
      if (c < 2) part[c * G + gg] = acc;
      else part[2 * G + gg * HD + c - 2] = acc;
    }
    cluster_arrive();                         // (2): partials published
    cluster_wait();

    // merge of the output slice over the C blocks, in rank order
#pragma unroll
    for (int k = 0; k < NOUT; ++k) {
      const int idx = o0 + ct + k * CT;
      if (idx < o1) {
        const int gg = idx / HD;
        float mr[kMaxCluster], lr[kMaxCluster], orr[kMaxCluster];
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
          if (r < C) {
            mr[r] = ld_peer(peer_addr(part + gg, r));
            lr[r] = ld_peer(peer_addr(part + G + gg, r));
            orr[r] = ld_peer(peer_addr(part + 2 * G + idx, r));
          }
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
          if (r < C) M = fmaxf(M, mr[r]);
        float L = 0.f, O = 0.f;
#pragma unroll
        for (int r = 0; r < kMaxCluster; ++r)
          if (r < C) {
            const float f = mr[r] == -INFINITY ? 0.f : exp2f(mr[r] - M);
            L = fmaf(f, lr[r], L);
            O = fmaf(f, orr[r], O);
          }
        a.a_out[(size_t)b * dm.qdim + kvh * G * HD + idx] =
            __float2bfloat16_rn(sigmoidf_(gate[k]) * (L > 0.f ? O / L : 0.f));
      }
    }
    cluster_arrive();                         // (3): peers' reads done
    cluster_wait();
  }

  // shutdown: after a timeout, wait (bounded) for the copies still in flight
  // before the shared memory is released
  __syncthreads();
  if (tid == 0 && *fail) {
    atomicOr(a.err, ERRBIT_TIMEOUT);
    const int hi = s_issued, lo2 = hi > kStages ? hi - kStages : 0;
    for (int i = lo2; i < hi; ++i)
      if (!mbar_wait(full + i % kStages, (uint32_t)((i / kStages) & 1))) break;
  }
}

template <int HD, int G>
size_t dec_smem() {
  constexpr int SK = (HD / 32) * kPanelBytes;
  constexpr int FLOATS = (G + 2) * HD + G * (HD + 2) + kCons * G * (HD + 2);
  return 1024 + (size_t)kStages * 2 * SK + (size_t)FLOATS * 4;
}

// Cluster size: 16 blocks where a 16-block cluster of this kernel fits on
// the GPU (a non-portable size), else the portable 8.
template <int HD, int G>
int dec_cluster(size_t smem) {
  static const int c = [smem] {
    auto k = attn_decode_kernel<HD, G>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
        cudaSuccess) {
      cudaGetLastError();
      return 8;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kMaxCluster, 1, 1);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kMaxCluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      return 8;
    }
    return kMaxCluster;
  }();
  return c;
}

template <int HD, int G>
void launch_dec_t(const DecAttnArgs& a, const CUtensorMap* maps,
                  cudaStream_t st) {
  const size_t smem = dec_smem<HD, G>();
  const int C = dec_cluster<HD, G>(smem);
  launch_k_cluster(attn_decode_kernel<HD, G>, dim3(C, a.dm.Hkv, a.B),
                   dim3(kDecThreads), smem, st, C, maps[0], maps[1], a);
}

template <int HD>
void launch_dec_hd(const DecAttnArgs& a, const CUtensorMap* maps,
                   cudaStream_t st) {
  switch (a.dm.Hq / a.dm.Hkv) {
    case 1: launch_dec_t<HD, 1>(a, maps, st); break;
    case 2: launch_dec_t<HD, 2>(a, maps, st); break;
    case 4: launch_dec_t<HD, 4>(a, maps, st); break;
    default: launch_dec_t<HD, 8>(a, maps, st); break;
  }
}

}  // namespace

int kv_tile_rows() { return DTK; }

void launch_attn_decode(const DecAttnArgs& a, const CUtensorMap* kv_maps,
                        cudaStream_t st) {
  switch (a.dm.hd) {
    case 64: launch_dec_hd<64>(a, kv_maps, st); break;
    case 128: launch_dec_hd<128>(a, kv_maps, st); break;
    default: launch_dec_hd<160>(a, kv_maps, st); break;
  }
}

}  // namespace dory
