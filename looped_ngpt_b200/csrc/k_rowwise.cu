// Row-wise kernels of the looped nGPT forward pass: embedding, RoPE table,
// the prefill nGPT update, greedy argmax and cache bookkeeping.  All are HBM/L2-bound and
// touch each element once.
#include "common.cuh"

namespace dory {

namespace {

// cos/sin of (n_ctx + t) * theta^(-2i/hd) for both attention types.  The
// angle is formed in double precision: at positions ~1e5 a float angle
// would be off by ~1e-2 rad.
__global__ void rope_table_kernel(float* table, const int* n_ctx, int T,
                                  int half, double th_swa, double th_full) {
  pdl_wait();
  pdl_trigger();
  const int total = 2 * T * half;
  const int p0 = *n_ctx;
  for (int id = blockIdx.x * blockDim.x + threadIdx.x; id < total;
       id += gridDim.x * blockDim.x) {
    const int type = id / (T * half);
    const int rem = id - type * T * half;
    const int t = rem / half, i = rem - t * half;
    const double theta = type ? th_full : th_swa;
    const double inv = pow(theta, -2.0 * i / (2.0 * half));
    double s, c;
    sincos((double)(p0 + t) * inv, &s, &c);
    table[2 * id] = (float)c;
    table[2 * id + 1] = (float)s;
  }
}

// x0 = N(E[tok]); one block per row.  For one-token calls (rope != null)
// block 0 also writes the RoPE cos/sin of position n_ctx for both attention
// types.
__global__ void embed_kernel(const int* tokens, const bf16* E, int d,
                             int vocab, float* s, bf16* s_bf, int* err,
                             float* rope, const int* n_ctx, int half,
                             double th_swa, double th_full) {
  __shared__ float red[32];
  const int row = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (row == 0) {
    if (rope) {
      const int p = *n_ctx;
      for (int id = threadIdx.x; id < 2 * half; id += blockDim.x) {
        const int type = id / half, i = id - type * half;
        const double inv = pow(type ? th_full : th_swa, -2.0 * i / (2.0 * half));
        double sn, c;
        sincos((double)p * inv, &sn, &c);
        rope[2 * id] = (float)c;
        rope[2 * id + 1] = (float)sn;
      }
    }
  }
  int tok = tokens[row];
  if (tok < 0 || tok >= vocab) {
    if (threadIdx.x == 0) atomicOr(err, ERRBIT_BOUNDS);
    tok = 0;
  }
  const bf16* e = E + (size_t)tok * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const float v = __bfloat162float(e[i]);
    ss += v * v;
  }
  const float inv = 1.f / fmaxf(sqrtf(block_sum(ss, red)), 1e-12f);
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const float v = __bfloat162float(e[i]) * inv;
    s[(size_t)row * d + i] = v;
    s_bf[(size_t)row * d + i] = __float2bfloat16_rn(v);
  }
}

// The nGPT update of whole rows (see ngpt_update_row for the algebra), one
// row per block of d / (4 NV) threads: thread i holds the 4-element groups
// at 4i + k d / NV (k < NV) in registers from the first read to the store,
// so a row is read once and written once (16-byte accesses), with one block
// reduction of the norm terms in between.  h: h_S K-split partials of the
// sublayer output, gridDim.x rows apart.  NV = 2 needs d % 256 == 0 and
// d <= 8192; NV = 4 (d % 512 == 0 and d <= 2560: 160 threads at d = 2560)
// halves the block so that four rows per SM are in flight instead of three.
// MIXED: rows carry their own loop counts (row_loops non-null); the plain
// variant has no per-row test at all.
template <bool MIXED, int NV>
__device__ __forceinline__ void update_row_body(
    const float* s_in, const float* h, const float* alpha, float* s_out,
    bf16* s_bf, float* x_buf, int reinject0, int d, int h_S,
    const int* row_loops, int T, int upd_loop, int rj_loop) {
  __shared__ float red[7 * 32];
  const size_t o = (size_t)blockIdx.x * d;
  const size_t hs = (size_t)gridDim.x * d;
  const int part = d / NV;
  pdl_wait();
  // rows with their own loop counts (uniform over the block: one row); a
  // row sitting out this loop keeps its state
  const int rj = MIXED ? row_reinject(row_loops, blockIdx.x / T, upd_loop,
                                      rj_loop, reinject0)
                       : reinject0;
  const bool frozen = MIXED && rj < 0;
  const int reinject = frozen ? RJ_NONE : rj;
  const bool next = reinject == RJ_NEXT;
  float4 sv[NV], av[NV], hv[NV], xv[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = 4 * threadIdx.x + k * part;
    sv[k] = *reinterpret_cast<const float4*>(s_in + o + i);
    av[k] = frozen ? make_float4(0.f, 0.f, 0.f, 0.f)
                   : *reinterpret_cast<const float4*>(alpha + i);
    hv[k] = frozen ? sv[k] : *reinterpret_cast<const float4*>(h + o + i);
    xv[k] = next ? *reinterpret_cast<const float4*>(x_buf + o + i)
                 : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  for (int p = 1; p < (frozen ? 1 : h_S); ++p)
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const float4 t = *reinterpret_cast<const float4*>(h + p * hs + o + 4 * threadIdx.x +
                                                        k * part);
      hv[k].x += t.x; hv[k].y += t.y; hv[k].z += t.z; hv[k].w += t.w;
    }
  pdl_trigger();
  float r[7] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  auto acc = [&](float s, float a, float hh, float x) {
    const float as = (1.f - a) * s, ah = a * hh;
    r[0] += hh * hh;
    r[1] += as * as;
    r[2] += as * ah;
    r[3] += ah * ah;
    r[4] += as * x;
    r[5] += ah * x;
    r[6] += x * x;
  };
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    acc(sv[k].x, av[k].x, hv[k].x, xv[k].x);
    acc(sv[k].y, av[k].y, hv[k].y, xv[k].y);
    acc(sv[k].z, av[k].z, hv[k].z, xv[k].z);
    acc(sv[k].w, av[k].w, hv[k].w, xv[k].w);
  }
  block_sum_n<7>(r, red);
  const float inv_h = 1.f / fmaxf(sqrtf(r[0]), 1e-12f);
  const float tt = r[1] + 2.f * r[2] * inv_h + r[3] * inv_h * inv_h;
  const float inv_t = 1.f / fmaxf(sqrtf(fmaxf(tt, 0.f)), 1e-12f);
  float inv_u = 1.f;
  if (next) {
    const float dot = (r[4] + r[5] * inv_h) * inv_t;
    inv_u = 1.f / fmaxf(sqrtf(fmaxf(1.f + 2.f * dot + r[6], 0.f)), 1e-12f);
  }
  auto upd = [&](float s, float a, float hh, float x, float* xs) {
    float v = ((1.f - a) * s + a * hh * inv_h) * inv_t;
    if (reinject == RJ_FIRST) *xs = v;
    if (next) v = (v + x) * inv_u;
    return v;
  };
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = 4 * threadIdx.x + k * part;
    float4 xo, vo;
    vo.x = upd(sv[k].x, av[k].x, hv[k].x, xv[k].x, &xo.x);
    vo.y = upd(sv[k].y, av[k].y, hv[k].y, xv[k].y, &xo.y);
    vo.z = upd(sv[k].z, av[k].z, hv[k].z, xv[k].z, &xo.z);
    vo.w = upd(sv[k].w, av[k].w, hv[k].w, xv[k].w, &xo.w);
    if (reinject == RJ_FIRST && x_buf) *reinterpret_cast<float4*>(x_buf + o + i) = xo;
    if (s_out) *reinterpret_cast<float4*>(s_out + o + i) = vo;
    if (s_bf) {
      uint2 u;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(vo.x, vo.y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(vo.z, vo.w);
      u.x = *reinterpret_cast<const uint32_t*>(&lo);
      u.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(s_bf + o + i) = u;
    }
  }
}

template <bool MIXED>
__global__ void update_rows_kernel(const float* s_in, const float* h,
                                   const float* alpha, float* s_out,
                                   bf16* s_bf, float* x_buf, int reinject0,
                                   int d, int h_S, const int* row_loops, int T,
                                   int upd_loop, int rj_loop) {
  update_row_body<MIXED, 2>(s_in, h, alpha, s_out, s_bf, x_buf, reinject0, d,
                            h_S, row_loops, T, upd_loop, rj_loop);
}

// d = 2560: 160 threads, four blocks (rows) per SM without spills
template <bool MIXED>
__global__ void __launch_bounds__(160, 4)
update_rows_wide_kernel(const float* s_in, const float* h, const float* alpha,
                        float* s_out, bf16* s_bf, float* x_buf, int reinject0,
                        int d, int h_S, const int* row_loops, int T,
                        int upd_loop, int rj_loop) {
  update_row_body<MIXED, 4>(s_in, h, alpha, s_out, s_bf, x_buf, reinject0, d,
                            h_S, row_loops, T, upd_loop, rj_loop);
}

// Lowest index among the maxima; NaN entries never win.
__device__ __forceinline__ void better(float& v, int& i, float cv, int ci) {
  if (cv > v || (cv == v && ci < i)) { v = cv; i = ci; }
}

__device__ void block_argmax(float v, int i, int* out) {
  __shared__ float sv[32];
  __shared__ int si[32];
  for (int o = 16; o > 0; o >>= 1) {
    const float ov = __shfl_xor_sync(0xffffffffu, v, o);
    const int oi = __shfl_xor_sync(0xffffffffu, i, o);
    better(v, i, ov, oi);
  }
  const int w = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) { sv[w] = v; si[w] = i; }
  __syncthreads();
  if (threadIdx.x == 0) {
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    for (int k = 0; k < (int)(blockDim.x >> 5); ++k) better(bv, bi, sv[k], si[k]);
    *out = bi == 0x7fffffff ? 0 : bi;
  }
}

// Also advances the cache length by T (block 0) when n_ctx != null: the
// attention of every layer of this call has finished reading it.
__global__ void argmax_partials_kernel(const float* val, const int* idx,
                                       int n, int* out, int* n_ctx, int T) {
  const int b = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  if (n_ctx && b == 0 && threadIdx.x == 0) *n_ctx += T;
  float v = -INFINITY;
  int i = 0x7fffffff;
  for (int k = threadIdx.x; k < n; k += blockDim.x)
    better(v, i, val[b * n + k], idx[b * n + k]);
  block_argmax(v, i, out + b);
}

__global__ void argmax_rows_kernel(const float* z, int V, int* out) {
  pdl_wait();
  pdl_trigger();
  const size_t r = blockIdx.x;
  float v = -INFINITY;
  int i = 0x7fffffff;
  for (int k = threadIdx.x; k < V; k += blockDim.x) better(v, i, z[r * V + k], k);
  block_argmax(v, i, out + r);
}

// SplitMix64 output function (Steele, Lea and Flood, 2014).
__device__ __forceinline__ uint64_t splitmix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Seeded synthetic cache entries for positions [p_lo, p_hi) of one slot:
// entry (kind, block, slot, b, kvh, pos, j) is the SplitMix64 counter
// generator's uniform u scaled to (2u - 1) * c_kind and rounded to bf16.
__global__ void fill_kv_kernel(KVSlot kv, CacheGeo g, int B, int Hkv, int hd,
                               int p_lo, int p_hi, int block, int slot,
                               uint64_t seed, float ck, float cv) {
  const int np = p_hi - p_lo;
  const long total = (long)B * Hkv * np * hd;
  for (long id = blockIdx.x * (long)blockDim.x + threadIdx.x; id < total;
       id += (long)gridDim.x * blockDim.x) {
    const int j = (int)(id % hd);
    long r = id / hd;
    const int pos = p_lo + (int)(r % np);
    r /= np;
    const int kvh = (int)(r % Hkv), b = (int)(r / Hkv);
    const size_t off = kv_index(kv, g, Hkv, hd, b, kvh, pos) + j;
#pragma unroll
    for (int kind = 0; kind < 2; ++kind) {
      uint64_t c = (uint64_t)kind;
      c = c * 64 + (uint64_t)block;
      c = c * 8 + (uint64_t)slot;
      c = c * 4096 + (uint64_t)b;
      c = c * 64 + (uint64_t)kvh;
      c = c * (1ull << 20) + (uint64_t)pos;
      c = c * 512 + (uint64_t)j;
      const uint64_t z = splitmix64(seed + c);
      const float u = __fmul_rn((float)(z >> 40), 0x1p-24f);
      const float x = __fmul_rn(__fsub_rn(__fmul_rn(2.f, u), 1.f), kind ? cv : ck);
      (kind ? kv.V : kv.K)[off] = __float2bfloat16_rn(x);
    }
  }
}

// Copy positions [p_lo, p_hi) of sequence src_b of one layer slot into every
// sequence of the same layer slot of another cache (rings and pages are
// addressed through each cache's own geometry); 16 bytes per thread.
__global__ void copy_prefix_kernel(KVSlot src, CacheGeo gs, int src_b,
                                   KVSlot dst, CacheGeo gd, int B_dst, int Hkv,
                                   int hd, int p_lo, int p_hi) {
  const int vec = hd / 8, np = p_hi - p_lo;
  const long total = (long)B_dst * Hkv * np * vec;
  for (long id = blockIdx.x * (long)blockDim.x + threadIdx.x; id < total;
       id += (long)gridDim.x * blockDim.x) {
    const int v = (int)(id % vec);
    long r = id / vec;
    const int pos = p_lo + (int)(r % np);
    r /= np;
    const int kvh = (int)(r % Hkv), b = (int)(r / Hkv);
    const size_t so = kv_index(src, gs, Hkv, hd, src_b, kvh, pos) + v * 8;
    const size_t dof = kv_index(dst, gd, Hkv, hd, b, kvh, pos) + v * 8;
    *reinterpret_cast<uint4*>(dst.K + dof) =
        *reinterpret_cast<const uint4*>(src.K + so);
    *reinterpret_cast<uint4*>(dst.V + dof) =
        *reinterpret_cast<const uint4*>(src.V + so);
  }
}

__global__ void set_nctx_kernel(int* n_ctx, int v) { *n_ctx = v; }

__global__ void advance_kernel(int* n_ctx, int T) {
  pdl_wait();
  pdl_trigger();
  *n_ctx += T;
}

__global__ void cache_init_kernel(int* n_ctx, int* bt, int total) {
  const int id = blockIdx.x * blockDim.x + threadIdx.x;
  if (id == 0) *n_ctx = 0;
  if (id < total) bt[id] = id;     // sequence b owns pages [b*P, (b+1)*P)
}

}  // namespace

void launch_rope_table(float* table, const CacheGeo& g, int T, int hd,
                       double theta_swa, double theta_full, cudaStream_t st) {
  const int total = 2 * T * (hd / 2);
  const int blocks = (total + 255) / 256;
  launch_k(rope_table_kernel, dim3(blocks < 1184 ? blocks : 1184), dim3(256), 0,
           st, table, (const int*)g.n_ctx, T, hd / 2, theta_swa, theta_full);
}

void launch_embed(const int* tokens, const bf16* E, int M, int d, float* s,
                  bf16* s_bf, int* err, int vocab, float* rope,
                  const int* n_ctx, int hd, double theta_swa,
                  double theta_full, cudaStream_t st) {
  launch_k(embed_kernel, dim3(M), dim3(256), 0, st, tokens, E, d, vocab, s,
           s_bf, err, rope, n_ctx, hd / 2, theta_swa, theta_full);
}

void launch_update_rows(const float* s_in, const float* h, const float* alpha,
                        float* s_out, bf16* s_bf, float* x_buf, int reinject,
                        int M, int d, cudaStream_t st, int h_S,
                        const int* row_loops, int T, int upd_loop,
                        int rj_loop) {
  const int Tp = T < 1 ? 1 : T;
  if (d % 512 == 0 && d <= 2560) {
    if (row_loops)
      launch_k(update_rows_wide_kernel<true>, dim3(M), dim3(d / 16), 0, st, s_in,
               h, alpha, s_out, s_bf, x_buf, reinject, d, h_S, row_loops, Tp,
               upd_loop, rj_loop);
    else
      launch_k(update_rows_wide_kernel<false>, dim3(M), dim3(d / 16), 0, st, s_in,
               h, alpha, s_out, s_bf, x_buf, reinject, d, h_S, row_loops, Tp,
               upd_loop, rj_loop);
  } else if (row_loops) {
    launch_k(update_rows_kernel<true>, dim3(M), dim3(d / 8), 0, st, s_in, h,
             alpha, s_out, s_bf, x_buf, reinject, d, h_S, row_loops, Tp,
             upd_loop, rj_loop);
  } else {
    launch_k(update_rows_kernel<false>, dim3(M), dim3(d / 8), 0, st, s_in, h,
             alpha, s_out, s_bf, x_buf, reinject, d, h_S, row_loops, Tp,
             upd_loop, rj_loop);
  }
}

void launch_argmax_partials(const float* val, const int* idx, int B, int n,
                            int* out, int* n_ctx, int T, cudaStream_t st) {
  launch_k(argmax_partials_kernel, dim3(B), dim3(256), 0, st, val, idx, n, out,
           n_ctx, T);
}

void launch_argmax_rows(const float* logits, int rows, int V, int* out,
                        cudaStream_t st) {
  launch_k(argmax_rows_kernel, dim3(rows), dim3(256), 0, st, logits, V, out);
}

void launch_fill_kv(const KVSlot& kv, const CacheGeo& g, int B, int Hkv,
                    int hd, int p_lo, int p_hi, int block, int slot,
                    uint64_t seed, float ck, float cv, cudaStream_t st) {
  if (p_hi <= p_lo) return;
  fill_kv_kernel<<<148 * 8, 256, 0, st>>>(kv, g, B, Hkv, hd, p_lo, p_hi, block,
                                          slot, seed, ck, cv);
}

void launch_set_nctx(int* n_ctx, int v, cudaStream_t st) {
  set_nctx_kernel<<<1, 1, 0, st>>>(n_ctx, v);
}

void launch_advance(int* n_ctx, int T, cudaStream_t st) {
  launch_k(advance_kernel, dim3(1), dim3(1), 0, st, n_ctx, T);
}

void launch_copy_prefix(const KVSlot& src, const CacheGeo& gs, int src_b,
                        const KVSlot& dst, const CacheGeo& gd, int B_dst,
                        int Hkv, int hd, int p_lo, int p_hi, cudaStream_t st) {
  if (p_hi <= p_lo) return;
  copy_prefix_kernel<<<148 * 4, 256, 0, st>>>(src, gs, src_b, dst, gd, B_dst,
                                               Hkv, hd, p_lo, p_hi);
}

void launch_cache_init(int* n_ctx, int* block_table, int B, int pages_per_seq,
                       cudaStream_t st) {
  const int total = B * pages_per_seq;
  cache_init_kernel<<<(total + 255) / 256 + 1, 256, 0, st>>>(n_ctx, block_table,
                                                             total);
}

}  // namespace dory
