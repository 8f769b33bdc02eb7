// Internal interface between the C-ABI host layer (dory_api.cu) and the
// sm_100a kernels.  Not installed; not part of the public ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>
#include <utility>

namespace dory {

typedef __nv_bfloat16 bf16;

// Launch with programmatic stream serialization (PDL) unless disabled.
bool pdl_enabled();
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block,
                            size_t smem, cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same with thread-block clusters of cluster_x blocks along x (grid.x
// a multiple of cluster_x).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k_cluster(void (*kernel)(KArgs...), dim3 grid,
                                    dim3 block, size_t smem, cudaStream_t st,
                                    int cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = cluster_x;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Host-side failure of a launcher that enqueued nothing (a tensor map that
// could not be encoded).  The launcher records it; every entry point clears
// the record before it enqueues work and returns DORY_ERR_CUDA if it is set
// afterwards.  Per host thread.
void note_host_failure(const char* what);
bool take_host_failure();

// Device error bits (or-ed into the status word the host reads back).
enum : int {
  ERRBIT_BOUNDS = 1,   // a position or index fell outside its buffer
  ERRBIT_TIMEOUT = 2,  // a bounded wait gave up
};

constexpr int kPage = 64;           // tokens per page of a full-attention cache
constexpr int kMaxHeadDim = 256;

struct Dims {
  int d, Hq, Hkv, hd, F, V;
  int qdim, kvdim, rows_qkvg;
  int window;
};

// One attention layer-slot of the KV cache.  ring = 1: sliding-window ring
// [B][Hkv][cap][hd]; ring = 0: pages [n_pages][Hkv][kPage][hd] reached
// through the cache's block table.
struct KVSlot {
  bf16* K;
  bf16* V;
  int ring;
  int cap;
};

struct CacheGeo {
  int* n_ctx;                // device: tokens held per sequence
  const int* block_table;    // device: [B][pages_per_seq]
  int pages_per_seq;
  int max_ctx;
};

__device__ __forceinline__ size_t kv_index(const KVSlot& s, const CacheGeo& g,
                                           int Hkv, int hd, int b, int kvh,
                                           int p) {
  if (s.ring) {
    int slot = p % s.cap;
    return ((size_t)(b * Hkv + kvh) * s.cap + slot) * hd;
  }
  int page = g.block_table[b * g.pages_per_seq + p / kPage];
  return (((size_t)page * Hkv + kvh) * kPage + (p % kPage)) * hd;
}

// ---------------------------------------------------------------- GEMV ----
enum GemvPro : int { PRO_BF16 = 0, PRO_UPDATE = 1 };
enum GemvEpi : int { EPI_F32 = 0, EPI_SWIGLU = 1, EPI_LMHEAD = 2 };
enum Reinject : int { RJ_NONE = 0, RJ_FIRST = 1, RJ_NEXT = 2 };

enum WFmt : int { WF_BF16 = 0, WF_MXFP8 = 1, WF_NVFP4 = 2 };

struct GemvArgs {
  const bf16* W;       // [N_rows, K] row-major (WF_BF16)
  int fmt;             // WFmt of W
  const uint8_t* Wq;   // WF_MXFP8: E4M3 [N][K]; WF_NVFP4: E2M1 pairs [N][K/2]
  const uint8_t* Ws;   // WF_MXFP8: E8M0 [N][K/32]; WF_NVFP4: E4M3 [N][K/16]
  const float* Wt;     // WF_NVFP4: tensor scale [1]
  int K;               // contraction length (multiple of 256 * S)
  int n_items;         // output rows (EPI_SWIGLU: pairs n, n + pair_off)
  int S;               // split-K factor: set to gemv_splits(*this)
  int B;               // batch rows, <= 8
  int pair_off;        // EPI_SWIGLU
  // prologue
  int pro;
  const bf16* xin;     // PRO_BF16: [B][xin_stride]
  int xin_stride;
  const float* s_in;   // PRO_UPDATE: current state [B][K]
  const float* h_in;   // sublayer output partials [h_S][B][K]
  int h_S;
  const float* alpha;  // [K]
  float* s_out;        // [B][K] (written by block 0)
  int reinject;
  float* x_buf;        // [B][K] input-block output (RJ_FIRST writes it)
  // epilogue
  int epi;
  float* out;          // EPI_F32: [S][B][n_items]; EPI_LMHEAD: logits
                       // [B][out_stride] or null
  int out_stride;
  bf16* out_bf;        // EPI_SWIGLU: [B][pair_off]
  const float* col_scale;   // EPI_LMHEAD: s_z [n_items]
  float* amax_val;     // EPI_LMHEAD: [B][gridDim]
  int* amax_idx;
  int* err;            // device status word (bounded-wait timeouts)
  // rows with their own loop counts (null: every row runs every loop)
  const int* row_loops; // [B] loops of each row
  int upd_loop;        // loop of the sublayer whose update the prologue
                       // applies (0: a non-recurrent block)
  int rj_loop;         // loop whose re-injection it applies (RJ_NEXT)
};
// K segments per row the launcher will use (outputs are [S][B][n] partials
// for EPI_F32; 1 for the other epilogues).
int gemv_splits(const GemvArgs& a);
int gemv_grid(const GemvArgs& a, int num_sms);
void launch_gemv(const GemvArgs& a, int grid, cudaStream_t st);

// Whole quantised matrix [N][K] to bf16 (e4m3 * 2^(e8m0 - 127), or
// e2m1 * e4m3 without the NVFP4 tensor scale; exact in bf16), the operand
// of the tensor-core GEMM for multi-token calls of quantised models.
void launch_dequant_bf16(int fmt, const uint8_t* Wq, const uint8_t* Ws, long N,
                         int K, bf16* out, cudaStream_t st);

// Decode rows [row0, row0 + nrows) of a quantised matrix to f32 (the values
// the GEMV multiplies: e4m3 * 2^(e8m0 - 127), or e2m1 * e4m3 without the
// NVFP4 tensor scale).  out [nrows][K].
void launch_dequant_rows(int fmt, const uint8_t* Wq, const uint8_t* Ws, int K,
                         int row0, int nrows, float* out, cudaStream_t st);

// ------------------------------------------------------------- rowwise ----
// RoPE cos/sin for positions n_ctx + t, t < T; table [2][T][hd/2][2].
void launch_rope_table(float* table, const CacheGeo& g, int T, int hd,
                       double theta_swa, double theta_full, cudaStream_t st);
// x0 = N(E[tok]) -> s (f32) and s_bf (bf16), rows M.  If rope != null
// (one-token calls) also writes the RoPE table [2][1][hd/2][2] for position
// n_ctx.
void launch_embed(const int* tokens, const bf16* E, int M, int d, float* s,
                  bf16* s_bf, int* err, int vocab, float* rope,
                  const int* n_ctx, int hd, double theta_swa,
                  double theta_full, cudaStream_t st);
// Rows that run their own loop counts: row b of a call takes part in loop t
// of the recurrent blocks iff t <= row_loops[b]; in the loops it sits out,
// its state is kept and it writes no K/V.  The effective re-injection of a
// pending update for row b: -1 = keep the state (the update belongs to a
// loop the row sits out), else RJ_NONE / RJ_FIRST / RJ_NEXT (RJ_NEXT drops
// to RJ_NONE when the row does not run loop rj_loop).
__device__ __forceinline__ int row_reinject(const int* row_loops, int b,
                                            int upd_loop, int rj_loop,
                                            int reinject) {
  if (!row_loops) return reinject;
  const int k = row_loops[b];
  if (upd_loop > k) return -1;
  if (reinject == RJ_NEXT && rj_loop > k) return RJ_NONE;
  return reinject;
}
__device__ __forceinline__ bool row_writes_kv(const int* row_loops, int b,
                                              int loop_t) {
  return !row_loops || loop_t <= row_loops[b];
}

// Prefill: s_new = N(s + alpha (N(h) - s)) per row (+ loop re-injection);
// rows b * T + t belong to sequence b (row_loops: see row_reinject).
void launch_update_rows(const float* s_in, const float* h, const float* alpha,
                        float* s_out, bf16* s_bf, float* x_buf, int reinject,
                        int M, int d, cudaStream_t st, int h_S = 1,
                        const int* row_loops = nullptr, int T = 1,
                        int upd_loop = 0, int rj_loop = 0);
// Final greedy argmax over [B][n] partials or full logits rows.
void launch_argmax_partials(const float* val, const int* idx, int B, int n,
                            int* out, int* n_ctx, int T, cudaStream_t st);
void launch_argmax_rows(const float* logits, int rows, int V, int* out,
                        cudaStream_t st);
void launch_advance(int* n_ctx, int T, cudaStream_t st);
void launch_set_nctx(int* n_ctx, int v, cudaStream_t st);
// Seeded synthetic K/V entries (SplitMix64 counter generator).
void launch_fill_kv(const KVSlot& kv, const CacheGeo& g, int B, int Hkv,
                    int hd, int p_lo, int p_hi, int block, int slot,
                    uint64_t seed, float ck, float cv, cudaStream_t st);
void launch_cache_init(int* n_ctx, int* block_table, int B, int pages_per_seq,
                       cudaStream_t st);
// K/V entries of positions [p_lo, p_hi) of sequence src_b of one layer slot
// -> the same positions of every sequence of a layer slot of another cache.
void launch_copy_prefix(const KVSlot& src, const CacheGeo& gs, int src_b,
                        const KVSlot& dst, const CacheGeo& gd, int B_dst,
                        int Hkv, int hd, int p_lo, int p_hi, cudaStream_t st);

// ----------------------------------------------------------- attention ----
struct AttnArgs {
  const bf16* q;       // [M][qdim], scaled by sqrt(hd) * log2(e)
  const float* gate;   // [M][qdim] sigmoid(g)
  int B, T;
  Dims dm;
  int window;          // 0 = full attention
  KVSlot kv; CacheGeo g;
  bf16* a_out;         // [M][qdim] = gate * attention output
  int* err;
};
// Prefill attention on the tcgen05 tensor cores.  kv_maps: this layer slot's K and V
// maps for 64-key tiles: K 64-dim boxes, K 32-dim boxes, V 64, V 32
// (make_map_2d with box_rows = pf_tile_keys()).  Ring capacities must be
// multiples of pf_tile_keys().
void launch_attn_prefill_tc(const AttnArgs& a, const CUtensorMap* kv_maps,
                            cudaStream_t st);
int pf_tile_keys();
// 2-D TMA map over a bf16 [rows][cols] matrix (row stride ld elements), box
// box_rows x box_cols with box_cols 64 (128-byte swizzle) or 32 (64-byte).
bool make_map_2d(CUtensorMap* m, const void* ptr, long rows, long cols,
                 long ld, int box_cols, int box_rows);
inline bool make_act_map(CUtensorMap* m, const void* ptr, long rows, long cols,
                         int box_cols, int box_rows) {
  return make_map_2d(m, ptr, rows, cols, cols, box_cols, box_rows);
}

// Decode (one token per sequence): RoPE/QK-norm/KV write, split-KV attention,
// split merge and gate in one kernel.
// A byte range of immutable data (weights) that a kernel asks the L2 cache
// to fetch ahead of the kernels that will read it.
struct L2Range {
  const void* p;
  long bytes;          // multiple of 16; p 16-byte aligned
};
constexpr int kMaxL2Ranges = 4;

struct DecAttnArgs {
  const float* qkvg;   // QKVG partials [S][B][rows_qkvg]
  int S, B;
  Dims dm;
  const float* s_q; const float* s_k;
  const float* rope;   // [hd/2][2] cos/sin of this layer's type at n_ctx
  float q_scale;
  int window;
  KVSlot kv; CacheGeo g;
  bf16* a_out;         // [B][qdim]
  int* err;
  // weights of the following projections, fetched into L2 while this
  // kernel (latency-bound at short context) leaves HBM idle
  L2Range l2pf[kMaxL2Ranges];
  const int* row_loops; // rows with their own loop counts, or null
  int loop_t;          // loop of this layer pass (0: non-recurrent)
};
// kv_maps: the TMA maps of this layer slot's K and V (make_kv_tile_map).
void launch_attn_decode(const DecAttnArgs& a, const CUtensorMap* kv_maps,
                        cudaStream_t st);
// Keys per decode-attention tile: ring capacities are multiples of it, and
// it is the box height of the KV tensor maps.
int kv_tile_rows();
// 2-D TMA map over a K or V cache buffer viewed as [rows][hd] bf16 (rows =
// ring slots or page rows), box kv_tile_rows() x 32 with the 64-byte swizzle.
bool make_kv_tile_map(CUtensorMap* m, const void* ptr, long rows, int hd);

// ---------------------------------------------------------------- GEMM ----
// C[M, N] (f32, row stride ldc) = A[M, K] (bf16, row stride lda) * W[N, K]^T
// optionally times col_scale[n], on tcgen05.  M, N any; K % 64 == 0.  When
// the output has fewer tiles than SMs (decode batches) and max_splits > 1,
// K is split: split z writes its partial to C + z * slab.  Returns the number
// of partials written (1 without a split).
// out_scale (device scalar or null) multiplies every product: the f32
// tensor scale of NVFP4 weights dequantised without it.
int launch_gemm_bf16(const bf16* A, int lda, const bf16* W, float* C, int ldc,
                     int M, int N, int K, const float* col_scale,
                     cudaStream_t st, int max_splits = 1, long slab = 0,
                     const float* out_scale = nullptr);
// Number of K-split partials launch_gemm_bf16 writes for this shape and
// max_splits (without a column scale).
int gemm_split_count(int M, int N, int K, int max_splits);
// m[M, F] = silu(A W_g^T) * (A W_u^T) as bf16, W = [W_g; W_u] (2F rows).
void launch_gemm_swiglu(const bf16* A, int lda, const bf16* W, bf16* m,
                        int ldm, int M, int F, int K, cudaStream_t st,
                        const float* out_scale = nullptr);
// Prefill q/k/v/gate projection with the RoPE, per-head L2 norm, scales,
// KV-cache write and gate sigmoid in the GEMM epilogue (one tile column per
// head).  A: bf16 [M][d] activations.
struct QkvGemmArgs {
  int M, T;
  Dims dm;
  const float* s_q; const float* s_k;
  const float* rope;   // this layer type's table [T][hd/2][2]
  float q_scale;
  KVSlot kv; CacheGeo g;
  bf16* q_out;         // [M][qdim]
  float* gate_out;     // [M][qdim]
  const int* row_loops; // rows with their own loop counts, or null
  int loop_t;          // loop of this layer pass (0: non-recurrent)
};
void launch_gemm_qkv(const bf16* A, int lda, const bf16* W,
                     const QkvGemmArgs& q, cudaStream_t st,
                     const float* out_scale = nullptr);
// ------------------------------------------------- speculative decoding ----
struct SpecArgs {
  const int* draft;     // [B][gamma+1]: last accepted token, then the drafts
  const int* target;    // [B][gamma+1]: the verifier's argmax per position
  const float* logits;  // [B][gamma+1][V]: verifier logits (inv_temp > 0)
  const float* uniform; // [B][gamma+1]: u_j for the test of draft j + 1,
                        // u_gamma for the one draw from the residual
  int B, gamma, V;
  float inv_temp;       // 1 / temperature; 0 = greedy
  int* r;               // [B] scratch: accepted drafts per sequence
  int* out;             // [B][gamma+1] emitted tokens (-1 past n_out)
  int* n_out;           // [1] tokens emitted per sequence
  int* n_ctx;           // device cache length, set to n0 + n_out
  int n0;
};
void launch_spec_accept(const SpecArgs& a, cudaStream_t st);
void launch_spec_transpose(const int* src, int* dst, int B, int G1,
                           cudaStream_t st);

// Device status word the tensor-core GEMM reports timeouts to.
void set_tc_error_word(int* err);

}  // namespace dory
