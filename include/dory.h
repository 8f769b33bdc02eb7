/*
 * dory.h -- C ABI of the B200 (sm_100a) elastic-depth forward pass of the
 * Dory1.0-4B looped normalized-GPT.
 *
 * What is computed (sources: the Dory1.0-4B pages):
 *   x0 = N(E[tok]); the input blocks map x0 to x; then for t = 1..k:
 *   u_t = N(s_{t-1} + x) with s_0 = x, s_t = N(F_theta(u_t)) where F_theta is
 *   the shared recurrent block; the output blocks run once; logits
 *   z = s_z * (W_lm s).  Effective depth 32 + 40k sublayers.
 *     -- "Dory1.0-4B: 循环归一化 GPT" (paper summary), 核心方法.
 *   Every sublayer updates s <- N(s + alpha (N(h) - s)) with per-channel
 *   alpha; the gated attention output and the SwiGLU activation are
 *   L2-normalised before their output projections.
 *     -- "Dory1.0-4B: A Looped Normalized-GPT" (paperlayer), §2 Architecture.
 *   Attention: GQA, sliding window 1024 (RoPE base 1e4) and full attention
 *   (RoPE base 1e7) interleaved 3:1, input-dependent sigmoid output gate.
 *     -- paper summary, 技术新颖性; MXFP8 explainer, hybrid-attention section.
 *   KV cache modes per_loop / last_loop: last_loop keeps one cache per
 *   recurrent attention layer and every loop overwrites it.
 *     -- paperlayer §6.1 Last-Loop KV Caching; MXFP8 explainer, last-loop.
 *
 * Conventions for every entry point:
 *   - Return 0 (DORY_OK) or a negative DORY_ERR_* code; dory_strerror()
 *     names it.  A failed call leaves caller buffers unspecified but the
 *     library state valid.  DORY_ERR_CUDA also covers a launch plan that
 *     could not be built on the host (a TMA descriptor the driver rejects);
 *     with DORY_DEBUG=1 in the environment the library names it on stderr.
 *   - Pointers prefixed d_ are device pointers (global memory of the current
 *     device); others are host pointers.  The caller allocates and owns every
 *     device buffer (weights, cache, workspace, outputs); the library keeps
 *     non-owning pointers plus small host-side plans.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued asynchronously; no entry point synchronises the device except
 *     dory_sync_status().
 */
#ifndef DORY_H_
#define DORY_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DORY_OK 0
#define DORY_ERR_ARG (-1)         /* null pointer, bad size, bad name/shape  */
#define DORY_ERR_UNSUPPORTED (-2) /* shape or format not compiled in         */
#define DORY_ERR_CACHE (-3)       /* kv_mode / loop count / context overflow */
#define DORY_ERR_CUDA (-4)        /* a CUDA call or launch failed            */
#define DORY_ERR_TIMEOUT (-5)     /* a bounded device wait gave up           */
#define DORY_ERR_WORKSPACE (-6)   /* workspace too small                     */
#define DORY_ERR_DEVICE (-7)      /* a device-side check recorded an error   */

typedef enum { DORY_KV_PER_LOOP = 0, DORY_KV_LAST_LOOP = 1 } dory_kv_mode;
typedef enum { DORY_W_BF16 = 0, DORY_W_MXFP8 = 1, DORY_W_NVFP4 = 2 } dory_wfmt;

/* Model shape.  A block is an attention sublayer followed by an MLP
 * sublayer; blocks are numbered 0..n_blocks-1 in execution order (input,
 * recurrent, output).  layer_types[i] = 0 (sliding window) or 1 (full).
 * Requirements (else DORY_ERR_UNSUPPORTED): head_dim in {64, 128, 160},
 * n_q_heads % n_kv_heads == 0 with at most 8 query heads per KV head, d,
 * ffn and n_q_heads*head_dim multiples of 256, vocab and the q/k/v/gate row
 * count multiples of 128, at least one input and one recurrent block. */
typedef struct {
  int d, n_q_heads, n_kv_heads, head_dim, ffn, vocab;
  int n_in_blocks, n_rec_blocks, n_out_blocks;
  const uint8_t* layer_types; /* host array of n_blocks entries (copied) */
  int swa_window;
  double rope_theta_swa, rope_theta_full;
  int wfmt;                   /* dory_wfmt of the block projections      */
} dory_config;

/* Quantised checkpoints (wfmt = DORY_W_MXFP8 / DORY_W_NVFP4; MXFP8 explainer
 * page, deployment section: W8A16, group 32; paper summary, 前置知识: NVFP4 =
 * E2M1 values with E4M3 scales): each block projection "blk<i>.<w>" is
 * replaced by
 *   "blk<i>.<w>.q"  uint8 codes: MXFP8 E4M3 [N, K]; NVFP4 E2M1 pairs
 *                   [N, K/2] (element 2j in bits 0-3, 2j+1 in bits 4-7)
 *   "blk<i>.<w>.s"  uint8 scales: MXFP8 E8M0 [N, K/32]; NVFP4 E4M3 [N, K/16]
 *   "blk<i>.<w>.t"  f32 [1] per-tensor scale (NVFP4 only)
 * with w = e4m3(q) * 2^(s - 127), or e2m1(q) * e4m3(s) * t.  Embedding and
 * LM head stay BF16.  One-token calls of up to 8 sequences decode the
 * weights in registers inside the GEMV; other calls (prefill, batches over
 * 8) decode each projection to bf16 in the workspace (exact: the products
 * have at most 8 significant bits) just before its tensor-core GEMM, which
 * applies the NVFP4 tensor scale t to its products.
 *
 * One named weight tensor in device memory (non-owning).  Names and shapes
 * (row-major, K = contraction axis last):
 *   "embed"  bf16 [vocab, d]       "lm_head" bf16 [vocab, d]
 *   "s_z"    f32  [vocab]
 *   "blk<i>.w_qkvg"  bf16 [2*Hq*h + 2*Hkv*h, d]  rows: q, k, v, gate
 *   "blk<i>.s_q"     f32 [Hq, h]     "blk<i>.s_k" f32 [Hkv, h]
 *   "blk<i>.w_o"     bf16 [d, Hq*h]  "blk<i>.alpha_a" f32 [d]
 *   "blk<i>.w_gu"    bf16 [2*ffn, d] rows: gate then up
 *   "blk<i>.w_down"  bf16 [d, ffn]   "blk<i>.alpha_m" f32 [d]
 * alpha, s_q, s_k, s_z are the effective values used in the forward pass.
 * Every device pointer must be 16-byte aligned. */
typedef struct {
  const char* name;
  const void* d_ptr;
  int64_t bytes;
} dory_tensor;

typedef struct dory_model dory_model;
typedef struct dory_cache dory_cache;

/* Validate the config and the weight table and build the host-side plan.
 * Every tensor listed above must be present with exactly its byte size.
 * No device memory is allocated; no kernel runs.  *out is released with
 * dory_free().  Errors: DORY_ERR_ARG (missing/mis-sized tensor, bad shape),
 * DORY_ERR_UNSUPPORTED (wfmt other than BF16, head_dim too large). */
int dory_init_weights(const dory_config* cfg, const dory_tensor* tensors,
                      int n_tensors, dory_model** out);

/* Bytes of device memory a KV cache needs for `batch` sequences of up to
 * `max_ctx` tokens, calls of up to `max_chunk` tokens per sequence, and (in
 * per_loop mode) up to `max_loops` loops.  The two modes are the pages'
 * recurrent KV-cache modes: per_loop keeps one cache per loop of every
 * recurrent attention layer, last_loop one cache per recurrent attention
 * layer that every loop overwrites, so its footprint equals the k = 1
 * footprint at any k ("Dory1.0-4B: A Looped Normalized-GPT", §6.1
 * Last-Loop KV Caching; MXFP8 explainer page, "循环 + KV 缓存" section).
 * Input and output blocks keep one cache each in both modes.  Layout: a small header, the full
 * attention layers as 64-token pages behind a block table, the
 * sliding-window layers as rings of min(max_ctx, window + max_chunk - 1)
 * positions rounded up to a multiple of 64 (the attention kernels' key
 * tiles never wrap a ring).  In last_loop mode the size does not depend on
 * max_loops. */
int dory_kv_cache_bytes(const dory_model* m, int batch, int max_ctx,
                        int max_chunk, int max_loops, int kv_mode,
                        int64_t* bytes);

/* Bind a caller-owned device buffer (>= dory_kv_cache_bytes, 256-byte
 * aligned) as an empty cache of the layout above (paperlayer §6.1;
 * sliding-window layers keep only their window, paper summary, 技术新颖性)
 * and enqueue its initialisation on `stream`:
 * the length and block table are set and every K/V row is zeroed (attention
 * tiles also read rows no token has written yet; their weights are 0 and
 * their contents must be finite).  The kv_mode is fixed for the life of the
 * cache. */
int dory_kv_cache_bind(dory_model* m, void* d_buf, int64_t bytes, int batch,
                       int max_ctx, int max_chunk, int max_loops, int kv_mode,
                       void* stream, dory_cache** out);

/* Tokens currently held per sequence (host mirror; all sequences of a cache
 * advance together). */
int dory_cache_length(const dory_cache* c, int* n_ctx);

/* Forget all cached tokens (per_loop caches also forget their loop count). */
int dory_cache_reset(dory_cache* c, void* stream);

/* Input generation for long-context workloads (not a step of the method):
 * make every sequence of the cache hold n_ctx tokens whose K/V entries are
 * seeded synthetic values, entry (kind K=0/V=1, block i, slot, b, kv head,
 * position, dim j) = bf16((2u - 1) * c_kind) with u the 24-bit uniform of
 * SplitMix64(seed + counter) and c_K = sqrt(3 / head_dim), c_V =
 * sqrt(3 / d); counter = ((((((kind*64 + i)*8 + slot)*4096 + b)*64 + kvh)
 * *2^20 + pos)*512 + j), slot = loop t (1-based) for per_loop recurrent
 * blocks and 0 otherwise.  Sliding-window layers receive only the positions
 * their ring keeps.  Replaces the cache contents; a per_loop cache forgets
 * its loop count.  Errors: DORY_ERR_ARG (n_ctx > max_ctx), DORY_ERR_CUDA. */
int dory_cache_fill_synthetic(dory_model* m, dory_cache* c, int n_ctx,
                              uint64_t seed, void* stream);

/* Prefix caching (long-context serving: a shared prompt prefix is computed
 * once and reused; the MXFP8 explainer page, deployment section, serves
 * contexts up to 256K): make every sequence of `dst` hold the first
 * n_tokens positions of sequence src_b of `src`, as if dst had prefilled
 * them itself; dst's length becomes n_tokens (its older contents are
 * dropped).  Full-attention layers copy every position; sliding-window
 * layers the window's last W - 1 positions that later queries can see.
 * Both caches must belong to the same model and kv_mode; a per_loop
 * source's loop count carries over (dst max_loops must hold it).  Errors:
 * DORY_ERR_ARG; DORY_ERR_CACHE (mode mismatch, n_tokens beyond the source's
 * length or dst's max_ctx, or a source ring that has already overwritten
 * positions the window still needs); DORY_ERR_CUDA.  Enqueued on
 * `stream`: order it after the source's writes and before dst's next call. */
int dory_cache_copy_prefix(dory_model* m, dory_cache* dst,
                           const dory_cache* src, int src_b, int n_tokens,
                           void* stream);

/* Workspace bytes for calls of `batch` sequences x up to `max_chunk`
 * tokens.  The workspace holds activations only; its contents between
 * calls are meaningless except for dory_copy_state(). */
int dory_workspace_bytes(const dory_model* m, int batch, int max_chunk,
                         int64_t* bytes);

/* Append T tokens per sequence (d_tokens int32 [B, T], row-major) and run
 * the looped forward pass over them with `n_loops` recurrent loops: the
 * input blocks once, the shared recurrent blocks n_loops times with the
 * re-injection u_t = N(s_{t-1} + x), the output blocks once, then the
 * logits (paper summary, 核心方法; the loop count is a per-request runtime
 * knob, MXFP8 explainer page, deployment section).  Inside a loop every
 * attention layer first writes the K/V of all T tokens to the slot the
 * kv_mode selects, then every query reads what each visible position holds
 * (paperlayer §6.1).
 * B must equal the bound batch, 1 <= T <= max_chunk, n_ctx + T <= max_ctx,
 * kv_mode must equal the cache's; a per_loop cache takes the loop count of
 * its first call and rejects any other (DORY_ERR_CACHE).
 * Outputs (either may be NULL): d_logits f32 [B, T, vocab] if logits_all
 * else [B, vocab] (last token); d_argmax int32 [B, T] or [B] (greedy, lowest
 * index on ties). */
int dory_prefill(dory_model* m, dory_cache* c, const int32_t* d_tokens, int B,
                 int T, int n_loops, int kv_mode, int logits_all,
                 float* d_logits, int32_t* d_argmax, void* d_workspace,
                 int64_t ws_bytes, void* stream);

/* One decode step: one token per sequence (d_tokens int32 [B]) through the
 * same looped forward pass as dory_prefill with T = 1 (paper summary,
 * 核心方法; in last_loop mode every loop's query reads the final-loop
 * entries of the earlier tokens, paperlayer §6.1).  Same rules as
 * dory_prefill.  The step is replayed from a CUDA graph once
 * its launch plan has been seen with the same pointers, B and n_loops. */
int dory_decode_step(dory_model* m, dory_cache* c, const int32_t* d_tokens,
                     int B, int n_loops, int kv_mode, float* d_logits,
                     int32_t* d_argmax, void* d_workspace, int64_t ws_bytes,
                     void* stream);

/* Self-speculative decoding ("Dory1.0-4B: A Looped Normalized-GPT", §6.2
 * Self-Speculative Decoding): the same weights at k_draft loops draft gamma
 * tokens one decode step at a time (greedy), then the k_verify-loop model
 * checks the last accepted token and the gamma drafts in one multi-token
 * pass, and rejection sampling decides how many drafts to keep.
 *   - d_last int32 [B]: the last accepted token of every sequence (not yet
 *     in the cache).  d_tokens_out int32 [B, gamma + 1] receives the
 *     emitted tokens, *n_out (host) their count n (1 <= n <= gamma + 1, the
 *     same for every sequence; entries past n are -1).  The cache advances
 *     by n: the emitted tokens except the last one, which is the next
 *     d_last.
 *   - temperature 0: greedy.  Draft j is kept while it equals the
 *     verifier's argmax, and the token after the kept drafts is the
 *     verifier's argmax there, so the output equals plain greedy decoding
 *     at k_verify loops.  temperature > 0: draft j is kept with probability
 *     p(draft j), p = softmax(logits / temperature) of the verifier, tested
 *     against d_uniform [B, gamma + 1] (values in [0, 1); entry j for draft
 *     j + 1); at the first rejection the token is drawn by inverse CDF with
 *     entry gamma from p restricted to the other tokens, and if all drafts
 *     are kept from p at the last position.  The output is distributed as
 *     sampling from the k_verify-loop model.  With several sequences every
 *     sequence advances by the smallest count; a sequence that kept more
 *     emits its own kept draft at the last position.
 *   - per_loop caches only, as on the pages (DORY_ERR_CACHE otherwise: in
 *     last_loop mode the tokens of one multi-token pass read each other's
 *     same-loop entries, so a verify pass would not reproduce one-token
 *     decoding).  The cache must be bound with max_loops >= k_verify and
 *     filled at k_verify loops (the draft reads the first k_draft slots,
 *     which the verifier's passes write).  The verifier rewrites every slot
 *     of the drafted positions before reading them.
 *   - The draft steps and the verify pass are replayed from CUDA graphs
 *     after their first use with the same pointers.  This entry point
 *     synchronises `stream` once, to read n.
 *   - Workspace: dory_spec_workspace_bytes.  BF16 weights only
 *     (DORY_ERR_UNSUPPORTED otherwise).  Errors as dory_prefill; gamma in
 *     1..15 with gamma + 1 <= max_chunk. */
int dory_spec_workspace_bytes(const dory_model* m, int B, int gamma,
                              int64_t* bytes);
int dory_spec_decode_step(dory_model* m, dory_cache* c, const int32_t* d_last,
                          int B, int gamma, int k_draft, int k_verify,
                          float temperature, const float* d_uniform,
                          int32_t* d_tokens_out, int* n_out,
                          void* d_workspace, int64_t ws_bytes, void* stream);

/* Test access to the acceptance step of dory_spec_decode_step alone, on
 * caller buffers: d_draft int32 [B, gamma + 1] (last token, then drafts),
 * d_target int32 [B, gamma + 1] (verifier argmax; greedy), d_logits f32
 * [B, gamma + 1, V] and d_uniform f32 [B, gamma + 1] (temperature > 0).
 * Writes d_tokens_out [B, gamma + 1] and d_scratch int32 [B + 2]
 * (d_scratch[0] = n). */
int dory_debug_spec_accept(const int32_t* d_draft, const int32_t* d_target,
                           const float* d_logits, const float* d_uniform,
                           int B, int gamma, int V, float temperature,
                           int32_t* d_tokens_out, int32_t* d_scratch,
                           void* stream);

/* Mixed loop counts in one batch (elastic depth per request: the loop count
 * is a per-request knob of a single checkpoint, paper summary, 研究动机 and
 * 核心方法): sequence b runs d_row_loops[b] recurrent loops (device int32
 * [B], each in 1..max_loops); the call runs max_loops loops, and in loop t
 * every sequence with d_row_loops[b] < t keeps its state and writes no K/V,
 * so each sequence computes exactly what a call with its own loop count
 * would.  Otherwise as dory_prefill / dory_decode_step with n_loops =
 * max_loops (a per_loop cache is bound to max_loops; each sequence must
 * keep its own count on every call, which the library cannot check).  The
 * decode step is replayed from a CUDA graph keyed by the pointers, the
 * d_row_loops buffer included (its contents may change between steps). */
int dory_prefill_mixed(dory_model* m, dory_cache* c, const int32_t* d_tokens,
                       int B, int T, const int32_t* d_row_loops, int max_loops,
                       int kv_mode, int logits_all, float* d_logits,
                       int32_t* d_argmax, void* d_workspace, int64_t ws_bytes,
                       void* stream);
int dory_decode_step_mixed(dory_model* m, dory_cache* c,
                           const int32_t* d_tokens, int B,
                           const int32_t* d_row_loops, int max_loops,
                           int kv_mode, float* d_logits, int32_t* d_argmax,
                           void* d_workspace, int64_t ws_bytes, void* stream);

/* Copy the final residual state s (input of the LM head, f32) of the last
 * call that used this workspace: [B, T, d] for a logits_all prefill, else
 * [B, d]. */
int dory_copy_state(const dory_model* m, const void* d_workspace, int B,
                    int T, int logits_all, float* d_out, void* stream);

/* Synchronise `stream` and report the device error word (bounded waits and
 * device-side checks): DORY_OK, DORY_ERR_TIMEOUT or DORY_ERR_DEVICE; a
 * failed synchronisation returns DORY_ERR_CUDA.  The word is cleared. */
int dory_sync_status(dory_model* m, void* stream);

/* Allocation-free decode step.  The pages have no counterpart: this entry
 * exists for callers that cannot call cudaMalloc (for example code running
 * under an allocator that owns all device memory, or a host process that
 * must not grow its device footprint after start-up), so they cannot provide
 * the workspace that dory_decode_step takes.  It runs the same kernels as
 * dory_decode_step with the workspace taken from a library-owned static
 * device array of DORY_STATIC_WS_BYTES bytes; every GPU that loads the
 * library holds that array until the process exits.  The caller still
 * passes the cache, the tokens and the outputs.
 *   - The first call on a device looks up that device's copy of the array
 *     (cudaGetSymbolAddress, with the device current); make that first call
 *     before any stream capture.
 *   - Returns DORY_ERR_WORKSPACE when dory_workspace_bytes(m, B, 1) exceeds
 *     DORY_STATIC_WS_BYTES; other errors as dory_decode_step.
 *   - Calls no cudaMalloc/cudaFree or other allocating routine (with
 *     profiling off, the default), and launches every kernel directly.
 *   - All calls share the one array: calls that may overlap on the GPU (on
 *     different streams, or from several threads) race and must be ordered
 *     by the caller.  Nothing in the array needs to start at zero: each call
 *     writes every word it reads before reading it. */
#define DORY_STATIC_WS_BYTES (8 << 20)
int dory_decode_step_static(dory_model* m, dory_cache* c,
                            const int32_t* d_tokens, int B, int n_loops,
                            int kv_mode, float* d_logits, int32_t* d_argmax,
                            void* stream);

/* Test and benchmark access to the projection GEMM used by prefill:
 * d_C f32 [M, N] (row-major) = d_A bf16 [M, K] (row stride lda >= K, a
 * multiple of 8) times d_W bf16 [N, K]^T, on the tcgen05 tensor cores.
 * K must be a multiple of 64; device pointers 16-byte aligned.  Enqueued on
 * `stream`; errors: DORY_ERR_ARG, DORY_ERR_CUDA (also when the operands'
 * TMA descriptors cannot be built, e.g. for a pointer that is not 16-byte
 * aligned; nothing is enqueued then); timeouts of its bounded waits are
 * reported by dory_sync_status of any model. */
int dory_debug_gemm_bf16(const void* d_A, int lda, const void* d_W,
                         float* d_C, int M, int N, int K, void* stream);

/* The same GEMM with the K split that decode batches use when the output has
 * fewer 128 x 256 tiles than the GPU has SMs: d_C holds max_splits slabs of
 * [M, N] f32, split z writes its partial sum over its K range to slab z, and
 * *n_partials (host) receives the number of slabs written; their sum is
 * A W^T.  Without a split (*n_partials = 1) slab 0 holds the product.
 * Errors as dory_debug_gemm_bf16, DORY_ERR_ARG also for max_splits < 1 or a
 * null n_partials. */
int dory_debug_gemm_bf16_split(const void* d_A, int lda, const void* d_W,
                               float* d_C, int M, int N, int K, int max_splits,
                               int* n_partials, void* stream);

/* Test access to the failure path of the bounded device waits: enqueue one
 * block whose thread waits on an mbarrier that nothing ever arrives on,
 * gives up after `polls` polls (1 <= polls <= 2^20; each poll returns
 * within microseconds) and records a timeout in the model's device status
 * word, then exits normally.  The next dory_sync_status() returns
 * DORY_ERR_TIMEOUT and clears the word; the context stays usable.  Errors:
 * DORY_ERR_ARG, DORY_ERR_CUDA. */
int dory_debug_bounded_wait(dory_model* m, int polls, void* stream);

/* Test access to the decode GEMV exactly as the forward pass runs it (same
 * kernel, same in-register weight decode, same K split): d_out = the block
 * projection `tensor` (e.g. "blk3.w_down"; "blk<i>.w_gu" as one [2F, K]
 * matrix) times the bf16 rows d_x [B, K] (1 <= B <= 8, 16-byte aligned),
 * written as *n_partials K-split partial slabs f32 [n][B][N] (d_out holds
 * max_partials slabs; at most 8 are written) whose sum is
 * the product.  Quantised models multiply the decoded weights (f16, exact)
 * by the activations rounded to f16, apply the group scale to each 8-term
 * sum and the NVFP4 tensor scale to the total; with a one-hot row x = e_k the
 * result is weight (n, k) times its scales, rounded once to f32, which is
 * how the tests compare the production decode bit for bit with the format
 * definitions.  Errors: DORY_ERR_ARG (bad name, B, alignment, or more
 * partials than max_partials), DORY_ERR_CUDA. */
int dory_debug_gemv(const dory_model* m, const char* tensor, const void* d_x,
                    int B, float* d_out, int max_partials, int* n_partials,
                    void* stream);

/* Test access to the in-register weight decode of quantised models: write
 * rows [row0, row0 + nrows) of block projection `tensor` (e.g.
 * "blk3.w_gu") as f32 [nrows, K] to d_out: e4m3(q) * 2^(s - 127) (MXFP8) or
 * e2m1(q) * e4m3(s) (NVFP4, without the tensor scale, which the GEMV applies
 * to its sums).  Both products are exact in f32.  Errors: DORY_ERR_ARG,
 * DORY_ERR_UNSUPPORTED (BF16 model). */
int dory_debug_dequant(const dory_model* m, const char* tensor, int row0,
                       int nrows, float* d_out, void* stream);

/* Per-kernel timing (tracing aid).  While enabled, every call launches its
 * kernels eagerly (no graph replay), each bracketed by CUDA events on the
 * call's stream, and records the kernel's algorithmic bytes (weights, KV
 * entries and activations it must move) and FLOPs. */
typedef struct {
  char name[32];      /* kernel class, e.g. "gemv_gateup", "attn_decode"   */
  int64_t launches;
  double total_ms;    /* summed event-measured durations                  */
  double bytes;       /* summed algorithmic bytes                          */
  double flops;       /* summed algorithmic FLOPs                          */
} dory_kernel_stat;

int dory_profile_enable(dory_model* m, int on);

/* Synchronise `stream`, aggregate the recorded launches by kernel class
 * into out[0..max) (*n = classes written) and clear the record. */
int dory_profile_read(dory_model* m, dory_kernel_stat* out, int max, int* n,
                      void* stream);

const char* dory_strerror(int code);
void dory_cache_free(dory_cache* c);
void dory_free(dory_model* m);

#ifdef __cplusplus
}
#endif
#endif /* DORY_H_ */
