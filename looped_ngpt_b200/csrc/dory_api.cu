// Host side of the C ABI declared in include/dory.h: validation, weight
// table, KV-cache and workspace layout, the per-call launch plan and CUDA
// graph replay of decode steps.
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <cmath>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <tuple>
#include <vector>

#include "dory.h"
#include "dory_internal.h"
#include "async_copy.cuh"

using namespace dory;

static __device__ int g_dory_status;   // or-ed ERRBIT_* from device checks

namespace dory {
namespace {
thread_local bool t_host_failure = false;
}
void note_host_failure(const char* what) {
  t_host_failure = true;
  const char* e = getenv("DORY_DEBUG");
  if (e && e[0] == '1') fprintf(stderr, "dory: %s could not be built\n", what);
}
bool take_host_failure() {
  const bool f = t_host_failure;
  t_host_failure = false;
  return f;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* e = getenv("DORY_NO_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}
}  // namespace dory

namespace {

// A block projection: BF16 rows, or quantised codes + scales (+ tensor scale).
struct QMat {
  const bf16* w = nullptr;
  const uint8_t* q = nullptr;
  const uint8_t* s = nullptr;
  const float* t = nullptr;
};

struct BlockW {
  const bf16 *w_qkvg, *w_o, *w_gu, *w_down;
  QMat m_qkvg, m_o, m_gu, m_down;
  const float *s_q, *s_k, *alpha_a, *alpha_m;
};

// (B, loops/T/logits_all, tokens, logits, argmax, workspace, row loop
// counts, cache): the cache comes last.
typedef std::tuple<int, int, const void*, const void*, const void*,
                   const void*, const void*, const void*> GraphKey;
constexpr size_t kKeyCache = std::tuple_size<GraphKey>::value - 1;

struct GraphEntry {
  int seen = 0;
  cudaGraphExec_t exec = nullptr;
};

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

struct dory_model {
  Dims dm;
  int wfmt = DORY_W_BF16;
  int n_in, n_rec, n_out, nblk;
  std::vector<uint8_t> ltype;
  double th_swa, th_full;
  const bf16* embed;
  const bf16* lm_head;
  const float* s_z;
  std::vector<BlockW> blk;
  int num_sms = 148;
  int device = 0;
  int* d_status = nullptr;
  bool use_graphs = true;
  cudaStream_t cap_stream = nullptr;
  std::map<GraphKey, GraphEntry> graphs;
  std::set<dory_cache*> caches;   // bound caches, detached by dory_free
  // per-kernel timing (dory_profile_enable)
  struct ProfRec {
    std::string name;
    cudaEvent_t a, b;
    double bytes, flops;
  };
  bool prof = false;
  std::vector<ProfRec> prof_recs;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_used = 0;
};

struct dory_cache {
  dory_model* m;
  int B, max_ctx, max_chunk, max_loops, kv_mode;
  int n_ctx = 0;
  int loops_bound = 0;
  int pages_per_seq;
  int swa_cap;
  int* d_nctx;
  int* d_block_table;
  std::vector<int> slot_base;   // per block: first entry in `slots`
  std::vector<KVSlot> slots;
  std::vector<CUtensorMap> kv_maps;   // per slot: decode maps of K, then V
  std::vector<CUtensorMap> pf_maps;   // per slot: prefill maps K64, K32, V64, V32
};

namespace {

bool is_rec(const dory_model* m, int i) {
  return i >= m->n_in && i < m->n_in + m->n_rec;
}

// Number of cache slots of block i: per_loop recurrent blocks keep one per
// loop; every other block keeps one.
int slots_of(const dory_model* m, int i, int kv_mode, int max_loops) {
  return (is_rec(m, i) && kv_mode == DORY_KV_PER_LOOP) ? max_loops : 1;
}

struct CacheLayout {
  size_t header, table, total;
  std::vector<size_t> k_off, v_off;
  std::vector<int> ring, cap;
  std::vector<int> base;
  int pages_per_seq, swa_cap;
};

CacheLayout cache_layout(const dory_model* m, int B, int max_ctx,
                         int max_chunk, int max_loops, int kv_mode) {
  CacheLayout L;
  const Dims& dm = m->dm;
  L.pages_per_seq = (max_ctx + kPage - 1) / kPage;
  // a multiple of the decode and prefill attention tiles (powers of two),
  // so that no tile wraps the ring
  const int tr = std::max(kv_tile_rows(), pf_tile_keys());
  L.swa_cap = (std::min(max_ctx, dm.window + max_chunk - 1) + tr - 1) / tr * tr;
  L.header = 256;
  L.table = align256((size_t)B * L.pages_per_seq * sizeof(int));
  size_t off = L.header + L.table;
  for (int i = 0; i < m->nblk; ++i) {
    L.base.push_back((int)L.k_off.size());
    const int n = slots_of(m, i, kv_mode, max_loops);
    for (int s = 0; s < n; ++s) {
      const bool full = m->ltype[i] == 1;
      const size_t per =
          full ? (size_t)B * L.pages_per_seq * dm.Hkv * kPage * dm.hd * 2
               : (size_t)B * dm.Hkv * L.swa_cap * dm.hd * 2;
      L.k_off.push_back(off);
      off += align256(per);
      L.v_off.push_back(off);
      off += align256(per);
      L.ring.push_back(full ? 0 : 1);
      L.cap.push_back(full ? 0 : L.swa_cap);
    }
  }
  L.total = off;
  return L;
}


struct WS {
  float *s0, *s1, *sfin, *x, *qkvg, *gate, *h, *lg,
      *rope, *amax_val;
  bf16 *s_bf, *a, *mact, *qb;
  bf16* wdq;          // quantised models, tensor-core calls: the projection
                      // being multiplied, dequantised to bf16
  int* amax_idx;
  size_t total;
};

constexpr int kMaxS = 8;
// K-split partials that a call may write into the f32 projection outputs
// (qkvg, h): decode batches that go through the tensor-core GEMM (one row
// tile) split K up to 16 ways, the GEMV at most kMaxS ways; multi-token
// calls split the W_o / W_down GEMMs only when their output has fewer tiles
// than the GPU has SMs (gemm_split_count, at most kMaxS).
int slabs_of(size_t M, int T) { return T == 1 && M <= 128 ? 16 : kMaxS; }
int h_slabs(const Dims& dm, int M, int T) {
  if (T == 1) return slabs_of(M, T);
  return std::max(gemm_split_count(M, dm.d, dm.qdim, kMaxS),
                  gemm_split_count(M, dm.d, dm.F, kMaxS));
}
constexpr int kArgmaxSlots = 2048;

WS ws_layout(const dory_model* m, int B, int T, char* base) {
  const Dims& dm = m->dm;
  const size_t M = (size_t)B * T;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  WS w;
  w.s0 = (float*)take(M * dm.d * 4);
  w.s1 = (float*)take(M * dm.d * 4);
  w.sfin = (float*)take(M * dm.d * 4);
  w.x = (float*)take(M * dm.d * 4);
  w.s_bf = (bf16*)take(M * dm.d * 2);
  // multi-token calls project q/k/v/gate inside the QKV GEMM epilogue
  w.qkvg = (float*)take(T == 1 ? slabs_of(M, T) * M * dm.rows_qkvg * 4 : 0);
  w.qb = (bf16*)take(M * dm.qdim * 2);
  w.gate = (float*)take(M * dm.qdim * 4);
  w.a = (bf16*)take(M * dm.qdim * 2);
  w.h = (float*)take((size_t)h_slabs(dm, (int)M, T) * M * dm.d * 4);
  w.mact = (bf16*)take(M * dm.F * 2);
  w.rope = (float*)take((size_t)2 * T * (dm.hd / 2) * 2 * 4);
  w.amax_val = (float*)take((size_t)B * kArgmaxSlots * 4);
  w.amax_idx = (int*)take((size_t)B * kArgmaxSlots * 4);
  w.lg = (float*)take(B > 8 ? (size_t)B * dm.V * 4 : 0);
  size_t wq = 0;
  if (m->wfmt != DORY_W_BF16 && !(T == 1 && B <= 8))
    wq = std::max(std::max((size_t)dm.rows_qkvg * dm.d, (size_t)dm.d * dm.qdim),
                  std::max((size_t)2 * dm.F * dm.d, (size_t)dm.d * dm.F)) * 2;
  w.wdq = (bf16*)take(wq);
  w.total = off;
  return w;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? DORY_OK : DORY_ERR_CUDA; }

}  // namespace

extern "C" {

int dory_profile_enable(dory_model* m, int on) {
  if (!m) return DORY_ERR_ARG;
  m->prof = on != 0;
  return DORY_OK;
}

int dory_profile_read(dory_model* m, dory_kernel_stat* out, int max, int* n,
                      void* stream) {
  if (!m || !n || (max > 0 && !out)) return DORY_ERR_ARG;
  *n = 0;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
    return DORY_ERR_CUDA;
  std::vector<dory_kernel_stat> agg;
  std::map<std::string, size_t> where;
  for (auto& r : m->prof_recs) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) continue;
    auto it = where.find(r.name);
    if (it == where.end()) {
      dory_kernel_stat st{};
      std::snprintf(st.name, sizeof(st.name), "%s", r.name.c_str());
      where[r.name] = agg.size();
      agg.push_back(st);
      it = where.find(r.name);
    }
    dory_kernel_stat& st = agg[it->second];
    st.launches += 1;
    st.total_ms += ms;
    st.bytes += r.bytes;
    st.flops += r.flops;
  }
  m->prof_recs.clear();
  m->ev_used = 0;
  cudaGetLastError();
  for (size_t i = 0; i < agg.size() && (int)i < max; ++i) out[(*n)++] = agg[i];
  return DORY_OK;
}

const char* dory_strerror(int code) {
  switch (code) {
    case DORY_OK: return "ok";
    case DORY_ERR_ARG: return "invalid argument";
    case DORY_ERR_UNSUPPORTED: return "unsupported shape or format";
    case DORY_ERR_CACHE: return "kv cache mismatch or overflow";
    case DORY_ERR_CUDA: return "CUDA error";
    case DORY_ERR_TIMEOUT: return "bounded device wait timed out";
    case DORY_ERR_WORKSPACE: return "workspace too small";
    case DORY_ERR_DEVICE: return "device-side check failed";
    default: return "unknown error";
  }
}

int dory_init_weights(const dory_config* cfg, const dory_tensor* tensors,
                      int n_tensors, dory_model** out) {
  if (!cfg || !out || (n_tensors > 0 && !tensors)) return DORY_ERR_ARG;
  *out = nullptr;
  const int d = cfg->d, Hq = cfg->n_q_heads, Hkv = cfg->n_kv_heads,
            hd = cfg->head_dim, F = cfg->ffn, V = cfg->vocab;
  if (d <= 0 || Hq <= 0 || Hkv <= 0 || hd <= 0 || F <= 0 || V <= 0)
    return DORY_ERR_ARG;
  if (cfg->n_in_blocks < 1 || cfg->n_rec_blocks < 1 || cfg->n_out_blocks < 0)
    return DORY_ERR_ARG;
  if (!cfg->layer_types || cfg->swa_window < 1) return DORY_ERR_ARG;
  if (!(cfg->rope_theta_swa > 1.0) || !(cfg->rope_theta_full > 1.0))
    return DORY_ERR_ARG;
  if (Hq % Hkv) return DORY_ERR_ARG;
  if (cfg->wfmt != DORY_W_BF16 && cfg->wfmt != DORY_W_MXFP8 &&
      cfg->wfmt != DORY_W_NVFP4)
    return DORY_ERR_UNSUPPORTED;
  const int G = Hq / Hkv;
  if (!(hd == 64 || hd == 128 || hd == 160) ||
      !(G == 1 || G == 2 || G == 4 || G == 8) || G * hd > 1024)
    return DORY_ERR_UNSUPPORTED;
  if (d % 256 || F % 256 || (Hq * hd) % 256 || V % 128 || d > 8192 ||
      F > 32768)
    return DORY_ERR_UNSUPPORTED;
  const int rows = 2 * Hq * hd + 2 * Hkv * hd;
  if (rows % 128) return DORY_ERR_UNSUPPORTED;

  dory_model* m = new dory_model();
  m->dm = Dims{d, Hq, Hkv, hd, F, V, Hq * hd, Hkv * hd, rows, cfg->swa_window};
  m->n_in = cfg->n_in_blocks;
  m->n_rec = cfg->n_rec_blocks;
  m->n_out = cfg->n_out_blocks;
  m->nblk = m->n_in + m->n_rec + m->n_out;
  m->ltype.assign(cfg->layer_types, cfg->layer_types + m->nblk);
  for (uint8_t t : m->ltype)
    if (t > 1) { delete m; return DORY_ERR_ARG; }
  m->th_swa = cfg->rope_theta_swa;
  m->th_full = cfg->rope_theta_full;
  m->wfmt = cfg->wfmt;

  std::map<std::string, std::pair<const void*, int64_t>> tab;
  for (int i = 0; i < n_tensors; ++i) {
    if (!tensors[i].name || !tensors[i].d_ptr ||
        ((uintptr_t)tensors[i].d_ptr & 15)) {
      delete m;
      return DORY_ERR_ARG;
    }
    tab[tensors[i].name] = {tensors[i].d_ptr, tensors[i].bytes};
  }
  bool ok = true;
  auto get = [&](const std::string& n, int64_t bytes) -> const void* {
    auto it = tab.find(n);
    if (it == tab.end() || it->second.second != bytes) {
      ok = false;
      return nullptr;
    }
    return it->second.first;
  };
  m->embed = (const bf16*)get("embed", (int64_t)V * d * 2);
  m->lm_head = (const bf16*)get("lm_head", (int64_t)V * d * 2);
  m->s_z = (const float*)get("s_z", (int64_t)V * 4);
  // block projections: BF16 `name`, or `name.q` / `name.s` (/ `name.t`)
  auto mat = [&](const std::string& n, int64_t N, int64_t K) {
    QMat q;
    if (cfg->wfmt == DORY_W_BF16) {
      q.w = (const bf16*)get(n, N * K * 2);
    } else if (cfg->wfmt == DORY_W_MXFP8) {
      q.q = (const uint8_t*)get(n + ".q", N * K);
      q.s = (const uint8_t*)get(n + ".s", N * K / 32);
    } else {
      q.q = (const uint8_t*)get(n + ".q", N * K / 2);
      q.s = (const uint8_t*)get(n + ".s", N * K / 16);
      q.t = (const float*)get(n + ".t", 4);
    }
    return q;
  };
  m->blk.resize(m->nblk);
  for (int i = 0; i < m->nblk; ++i) {
    const std::string p = "blk" + std::to_string(i) + ".";
    BlockW& b = m->blk[i];
    b.m_qkvg = mat(p + "w_qkvg", rows, d);
    b.m_o = mat(p + "w_o", d, (int64_t)Hq * hd);
    b.m_gu = mat(p + "w_gu", 2 * (int64_t)F, d);
    b.m_down = mat(p + "w_down", d, F);
    b.w_qkvg = b.m_qkvg.w;
    b.w_o = b.m_o.w;
    b.w_gu = b.m_gu.w;
    b.w_down = b.m_down.w;
    b.s_q = (const float*)get(p + "s_q", (int64_t)Hq * hd * 4);
    b.s_k = (const float*)get(p + "s_k", (int64_t)Hkv * hd * 4);
    b.alpha_a = (const float*)get(p + "alpha_a", (int64_t)d * 4);
    b.alpha_m = (const float*)get(p + "alpha_m", (int64_t)d * 4);
  }
  if (!ok) { delete m; return DORY_ERR_ARG; }

  if (cudaGetDevice(&m->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&m->num_sms, cudaDevAttrMultiProcessorCount,
                             m->device) != cudaSuccess ||
      cudaGetSymbolAddress((void**)&m->d_status, g_dory_status) != cudaSuccess) {
    delete m;
    return DORY_ERR_CUDA;
  }
  set_tc_error_word(m->d_status);
  const char* ng = getenv("DORY_NO_GRAPH");
  m->use_graphs = !(ng && ng[0] == '1');
  *out = m;
  return DORY_OK;
}

void dory_free(dory_model* m) {
  if (!m) return;
  for (dory_cache* c : m->caches) c->m = nullptr;   // caches may outlive m
  for (auto& kv : m->graphs)
    if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
  if (m->cap_stream) cudaStreamDestroy(m->cap_stream);
  for (cudaEvent_t e : m->ev_pool) cudaEventDestroy(e);
  delete m;
}

int dory_kv_cache_bytes(const dory_model* m, int batch, int max_ctx,
                        int max_chunk, int max_loops, int kv_mode,
                        int64_t* bytes) {
  if (!m || !bytes || batch < 1 || max_ctx < 1 || max_chunk < 1 ||
      max_chunk > max_ctx || (kv_mode != 0 && kv_mode != 1))
    return DORY_ERR_ARG;
  if (kv_mode == DORY_KV_PER_LOOP && max_loops < 1) return DORY_ERR_ARG;
  if (kv_mode == DORY_KV_LAST_LOOP) max_loops = 1;
  *bytes = (int64_t)cache_layout(m, batch, max_ctx, max_chunk, max_loops,
                                 kv_mode).total;
  return DORY_OK;
}

int dory_kv_cache_bind(dory_model* m, void* d_buf, int64_t bytes, int batch,
                       int max_ctx, int max_chunk, int max_loops, int kv_mode,
                       void* stream, dory_cache** out) {
  if (!out) return DORY_ERR_ARG;
  *out = nullptr;
  int64_t need = 0;
  int rc = dory_kv_cache_bytes(m, batch, max_ctx, max_chunk, max_loops,
                               kv_mode, &need);
  if (rc) return rc;
  if (!d_buf || ((uintptr_t)d_buf & 255) || bytes < need) return DORY_ERR_ARG;
  if (kv_mode == DORY_KV_LAST_LOOP) max_loops = 1;
  CacheLayout L = cache_layout(m, batch, max_ctx, max_chunk, max_loops, kv_mode);
  dory_cache* c = new dory_cache();
  c->m = m;
  c->B = batch;
  c->max_ctx = max_ctx;
  c->max_chunk = max_chunk;
  c->max_loops = max_loops;
  c->kv_mode = kv_mode;
  c->pages_per_seq = L.pages_per_seq;
  c->swa_cap = L.swa_cap;
  char* base = (char*)d_buf;
  c->d_nctx = (int*)base;
  c->d_block_table = (int*)(base + L.header);
  c->slot_base = L.base;
  for (size_t i = 0; i < L.k_off.size(); ++i) {
    const KVSlot kv{(bf16*)(base + L.k_off[i]), (bf16*)(base + L.v_off[i]),
                    L.ring[i], L.cap[i]};
    c->slots.push_back(kv);
    // rows of the [rows][hd] view: ring slots, or every page's rows
    const long rows = kv.ring ? (long)batch * m->dm.Hkv * kv.cap
                              : (long)batch * L.pages_per_seq * m->dm.Hkv * kPage;
    CUtensorMap mk, mv;
    if (!make_kv_tile_map(&mk, kv.K, rows, m->dm.hd) ||
        !make_kv_tile_map(&mv, kv.V, rows, m->dm.hd)) {
      delete c;
      return DORY_ERR_CUDA;
    }
    c->kv_maps.push_back(mk);
    c->kv_maps.push_back(mv);
    CUtensorMap pm[4];
    const int hd = m->dm.hd, tk = pf_tile_keys();
    if (!make_map_2d(&pm[0], kv.K, rows, hd, hd, 64, tk) ||
        !make_map_2d(&pm[1], kv.K, rows, hd, hd, 32, tk) ||
        !make_map_2d(&pm[2], kv.V, rows, hd, hd, 64, tk) ||
        !make_map_2d(&pm[3], kv.V, rows, hd, hd, 32, tk)) {
      delete c;
      return DORY_ERR_CUDA;
    }
    for (int k = 0; k < 4; ++k) c->pf_maps.push_back(pm[k]);
  }
  // finite contents everywhere: attention tiles also cover rows that no
  // token has written yet (their probabilities are 0, their values must not
  // be NaN)
  cudaMemsetAsync(base + L.header + L.table, 0, L.total - L.header - L.table,
                  (cudaStream_t)stream);
  launch_cache_init(c->d_nctx, c->d_block_table, batch, L.pages_per_seq,
                    (cudaStream_t)stream);
  if (cudaGetLastError() != cudaSuccess) { delete c; return DORY_ERR_CUDA; }
  m->caches.insert(c);
  *out = c;
  return DORY_OK;
}

int dory_cache_length(const dory_cache* c, int* n_ctx) {
  if (!c || !n_ctx) return DORY_ERR_ARG;
  *n_ctx = c->n_ctx;
  return DORY_OK;
}

int dory_cache_reset(dory_cache* c, void* stream) {
  if (!c || !c->m) return DORY_ERR_ARG;
  c->n_ctx = 0;
  c->loops_bound = 0;
  launch_cache_init(c->d_nctx, c->d_block_table, c->B, c->pages_per_seq,
                    (cudaStream_t)stream);
  return cuda_rc(cudaGetLastError());
}

void dory_cache_free(dory_cache* c) {
  if (!c) return;
  dory_model* m = c->m;
  if (!m) {             // its model was freed first
    delete c;
    return;
  }
  m->caches.erase(c);
  for (auto it = m->graphs.begin(); it != m->graphs.end();) {
    if (std::get<kKeyCache>(it->first) == (const void*)c) {
      if (it->second.exec) cudaGraphExecDestroy(it->second.exec);
      it = m->graphs.erase(it);
    } else {
      ++it;
    }
  }
  delete c;
}

int dory_workspace_bytes(const dory_model* m, int batch, int max_chunk,
                         int64_t* bytes) {
  if (!m || !bytes || batch < 1 || max_chunk < 1) return DORY_ERR_ARG;
  // the split-K slab count depends on the call's token count, so a shorter
  // call can need more bytes than a longer one: take the largest layout
  size_t mx = 0;
  for (int T = 1; T <= max_chunk; ++T)
    mx = std::max(mx, ws_layout(m, batch, T, nullptr).total);
  *bytes = (int64_t)mx;
  return DORY_OK;
}

}  // extern "C"

namespace {

// Brackets one launch with CUDA events when profiling is on.
struct Prof {
  dory_model* m;
  cudaStream_t st;
  long idx = -1;
  Prof(dory_model* mm, cudaStream_t s, const char* name, double bytes,
       double flops)
      : m(mm), st(s) {
    if (!m->prof) return;
    while (m->ev_pool.size() < m->ev_used + 2) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) return;
      m->ev_pool.push_back(e);
    }
    dory_model::ProfRec r{name, m->ev_pool[m->ev_used], m->ev_pool[m->ev_used + 1],
                          bytes, flops};
    m->ev_used += 2;
    cudaEventRecord(r.a, st);
    m->prof_recs.push_back(r);
    idx = (long)m->prof_recs.size() - 1;
  }
  ~Prof() {
    if (idx >= 0) cudaEventRecord(m->prof_recs[idx].b, st);
  }
};

double gemv_bytes(const GemvArgs& g, int rows) {
  // weight bytes per element: BF16 2, MXFP8 1 + 1/32, NVFP4 1/2 + 1/16
  const double per = g.fmt == WF_MXFP8 ? 1.0 + 1.0 / 32
                     : g.fmt == WF_NVFP4 ? 0.5 + 1.0 / 16 : 2.0;
  const double w = (double)rows * g.K * per;
  const double in = g.pro == PRO_UPDATE ? (double)g.B * g.K * 4 * (3 + g.h_S)
                                        : (double)g.B * g.K * 2;
  double out;
  if (g.epi == EPI_SWIGLU) out = (double)g.B * g.n_items * 2;
  else if (g.epi == EPI_LMHEAD) out = g.out ? (double)g.B * g.n_items * 4 : 0;
  else out = (double)g.S * g.B * g.n_items * 4;
  return w + in + out;
}

// Launches the GEMV; returns the number of K segments (partials) it writes.
int gemv_run(dory_model* m, const GemvArgs& g0, cudaStream_t st,
             const char* name, const QMat* qm = nullptr) {
  GemvArgs g = g0;
  g.err = m->d_status;
  g.fmt = WF_BF16;
  if (qm && !qm->w) {
    g.fmt = m->wfmt == DORY_W_MXFP8 ? WF_MXFP8 : WF_NVFP4;
    g.Wq = qm->q;
    g.Ws = qm->s;
    g.Wt = qm->t;
  }
  g.S = gemv_splits(g);
  const int grid = gemv_grid(g, m->num_sms);
  const int rows = g.epi == EPI_SWIGLU ? 2 * g.n_items : g.n_items;
  Prof p(m, st, name, gemv_bytes(g, rows), 2.0 * rows * g.K * g.B);
  launch_gemv(g, grid, st);
  return g.S;
}

// Returns the number of K-split partials written (C + z * M * ldc).
int gemm_run(dory_model* m, const bf16* A, int lda, const bf16* W, float* C,
             int ldc, int M, int N, int K, const float* scale,
             cudaStream_t st, const char* name, int max_splits = 1,
             const float* out_scale = nullptr) {
  Prof p(m, st, name,
         (double)M * K * 2 + (double)N * K * 2 + (double)M * N * 4,
         2.0 * M * N * K);
  return launch_gemm_bf16(A, lda, W, C, ldc, M, N, K, scale, st, max_splits,
                          (long)M * ldc, out_scale);
}

// BF16 operand of a projection for the tensor-core GEMM: the weights
// themselves, or (quantised models) their exact bf16 decode written to the
// workspace just before the GEMM that reads it.  The NVFP4 tensor scale is
// left out and applied by the GEMM to its products (*out_scale).
const bf16* gemm_weight(dory_model* m, const QMat& q, long N, long K, bf16* wdq,
                        cudaStream_t st, const float** out_scale) {
  *out_scale = nullptr;
  if (q.w) return q.w;
  const int fmt = m->wfmt == DORY_W_MXFP8 ? WF_MXFP8 : WF_NVFP4;
  const double per = fmt == WF_MXFP8 ? 1.0 + 1.0 / 32 : 0.5 + 1.0 / 16;
  Prof p(m, st, "dequant", (double)N * K * (per + 2.0), 0);
  launch_dequant_bf16(fmt, q.q, q.s, N, (int)K, wdq, st);
  *out_scale = q.t;
  return wdq;
}

struct CallCtx {
  dory_model* m;
  dory_cache* c;
  WS w;
  int B, T, M, n_loops, logits_all, n_ctx0;
  const int* tokens;
  float* logits;
  int* argmax;
  cudaStream_t st;
  const int* row_loops;   // device [B] per-sequence loop counts, or null
};

int slot_index(const dory_cache* c, int i, int t) {
  int idx = c->slot_base[i];
  if (is_rec(c->m, i) && c->kv_mode == DORY_KV_PER_LOOP) idx += t - 1;
  return idx;
}
KVSlot slot_for(const dory_cache* c, int i, int t) {
  return c->slots[slot_index(c, i, t)];
}

bool use_gemv(int B, int T) { return T == 1 && B <= 8; }

// Decode attention at short context reads a few MB and is bound by latency,
// leaving HBM idle: once its predecessor has finished, it asks L2 for a
// leading share of the gate and of the up rows of W_gu, which the gate/up
// GEMV then reads from L2.  Measured at batch 1, k = 2, 2048-token context
// (percent of the rows -> tok/s): 0 -> 306, 10 -> 310, 20 -> 313,
// 30 -> 307, 35 -> 301; W_o (whose GEMV loads it during the attention
// anyway) and W_down shares only cost.  Issued before the dependency wait
// the same prefetch slowed the step (it competes with the QKVG GEMV's own
// stream).  Above kL2pfMaxKvBytes of K/V per call the attention itself
// streams HBM and nothing is prefetched.  DORY_L2PF_WO / _GU / _DOWN
// (percent) override the shares.
constexpr double kL2pfMaxKvBytes = 64e6;
// A percentage from the environment as a fraction in [0, 1].
double env_fraction(const char* name, double dflt) {
  const char* e = getenv(name);
  const double v = e ? atof(e) / 100.0 : dflt;
  return v < 0.0 ? 0.0 : (v > 1.0 ? 1.0 : v);
}
void set_l2_prefetch(const dory_model* m, const BlockW& bw, L2Range* r) {
  const double f_o = env_fraction("DORY_L2PF_WO", 0.0);
  const double f_gu = env_fraction("DORY_L2PF_GU", 0.2);
  const double f_dn = env_fraction("DORY_L2PF_DOWN", 0.0);
  const Dims& dm = m->dm;
  // bytes per weight row of a projection with K inputs
  auto row_bytes = [&](const QMat& q, long K) -> long {
    if (q.w) return K * 2;
    return m->wfmt == DORY_W_MXFP8 ? K : K / 2;
  };
  auto base = [](const QMat& q) -> const char* {
    return q.w ? (const char*)q.w : (const char*)q.q;
  };
  const long ro = row_bytes(bw.m_o, dm.qdim);
  const long rg = row_bytes(bw.m_gu, dm.d);
  const long n_o = (long)(dm.d * f_o);
  const long n_g = (long)(dm.F * f_gu);
  r[0] = L2Range{base(bw.m_o), n_o * ro};
  r[1] = L2Range{base(bw.m_gu), n_g * rg};
  r[2] = L2Range{base(bw.m_gu) + (long)dm.F * rg, n_g * rg};
  const long rd = row_bytes(bw.m_down, dm.F);
  r[3] = L2Range{base(bw.m_down), (long)(dm.d * f_dn) * rd};
}

// Enqueue one forward pass: embedding, input blocks, n_loops passes of the
// recurrent blocks with re-injection, output blocks, LM head.
void enqueue_forward(const CallCtx& x) {
  dory_model* m = x.m;
  const Dims& dm = m->dm;
  const WS& w = x.w;
  const bool gemv = use_gemv(x.B, x.T);
  const CacheGeo geo{x.c->d_nctx, x.c->d_block_table, x.c->pages_per_seq,
                     x.c->max_ctx};
  const int half = dm.hd / 2;
  const float q_scale = sqrtf((float)dm.hd) * 1.4426950408889634f;
  if (x.T > 1) {
    Prof p(m, x.st, "rope_table", 16.0 * x.T * half, 0);
    launch_rope_table(w.rope, geo, x.T, dm.hd, m->th_swa, m->th_full, x.st);
  }
  {
    Prof p(m, x.st, "embed", (double)x.M * dm.d * 8, 0);
    launch_embed(x.tokens, m->embed, x.M, dm.d, w.s0, w.s_bf, m->d_status,
                 dm.V, x.T == 1 ? w.rope : nullptr,
                 geo.n_ctx, dm.hd, m->th_swa, m->th_full, x.st);
  }
  float* cur = w.s0;
  float* other = w.s1;
  const float* prev_alpha = nullptr;
  int prev_S = 1;
  const int slabs = slabs_of(x.M, x.T);       // K-split partials that fit

  std::vector<std::pair<int, int>> order;
  for (int i = 0; i < m->n_in; ++i) order.push_back({i, 0});
  for (int t = 1; t <= x.n_loops; ++t)
    for (int i = m->n_in; i < m->n_in + m->n_rec; ++i) order.push_back({i, t});
  for (int i = m->n_in + m->n_rec; i < m->nblk; ++i) order.push_back({i, 0});

  int prev_t = 0;        // loop of the previous layer pass (0: not recurrent)
  for (size_t k = 0; k < order.size(); ++k) {
    const int i = order[k].first, t = order[k].second;
    const int rj_loop = (i == m->n_in && t > 1) ? t : 0;
    const BlockW& bw = m->blk[i];
    int rj = RJ_NONE;
    if (i == m->n_in) rj = (t == 1) ? RJ_FIRST : RJ_NEXT;
    const bool full = m->ltype[i] == 1;
    const KVSlot kv = slot_for(x.c, i, t);

    // ---- attention sublayer -------------------------------------------
    int S_qkvg = 1;
    if (gemv) {
      GemvArgs g{};
      g.W = bw.w_qkvg; g.K = dm.d; g.n_items = dm.rows_qkvg; g.B = x.B;
      g.epi = EPI_F32;
      g.out = w.qkvg;
      if (k == 0) {
        g.pro = PRO_BF16; g.xin = w.s_bf; g.xin_stride = dm.d;
      } else {
        g.pro = PRO_UPDATE; g.s_in = cur; g.h_in = w.h; g.h_S = prev_S;
        g.alpha = prev_alpha; g.s_out = other; g.reinject = rj; g.x_buf = w.x;
        g.row_loops = x.row_loops; g.upd_loop = prev_t; g.rj_loop = rj_loop;
        std::swap(cur, other);
      }
      S_qkvg = gemv_run(m, g, x.st, "gemv_qkvg", &bw.m_qkvg);
    } else {
      if (k > 0) {
        Prof p(m, x.st, "update_rows", (double)x.M * dm.d * 14, 0);
        launch_update_rows(cur, w.h, prev_alpha, other, w.s_bf, w.x, rj, x.M,
                           dm.d, x.st, prev_S, x.row_loops, x.T, prev_t,
                           rj_loop);
        std::swap(cur, other);
      }
      const float* osc = nullptr;
      const bf16* Wqkvg = gemm_weight(m, bw.m_qkvg, dm.rows_qkvg, dm.d, w.wdq,
                                      x.st, &osc);
      if (x.T == 1) {
        // one partial: the attention cluster's owner warps sum the q/k/v
        // partials on the critical path before the cluster's first barrier;
        // at B = 64 a 5-way split saved 0.45 ms here and cost 1.2 ms there
        gemm_run(m, w.s_bf, dm.d, Wqkvg, w.qkvg, dm.rows_qkvg, x.M,
                 dm.rows_qkvg, dm.d, nullptr, x.st, "gemm_qkvg", 1, osc);
      } else {
        QkvGemmArgs qg{};
        qg.M = x.M; qg.T = x.T; qg.dm = dm; qg.s_q = bw.s_q; qg.s_k = bw.s_k;
        qg.rope = w.rope + (full ? (size_t)x.T * half * 2 : 0);
        qg.q_scale = q_scale; qg.kv = kv; qg.g = geo;
        qg.q_out = w.qb; qg.gate_out = w.gate;
        qg.row_loops = x.row_loops; qg.loop_t = t;
        Prof p(m, x.st, "gemm_qkv",
               (double)x.M * dm.d * 2 + (double)dm.rows_qkvg * dm.d * 2 +
                   (double)x.M * (dm.qdim * 6.0 + dm.kvdim * 4.0),
               2.0 * x.M * dm.rows_qkvg * dm.d);
        launch_gemm_qkv(w.s_bf, dm.d, Wqkvg, qg, x.st, osc);
      }
    }
    if (x.T == 1) {
      DecAttnArgs da{};
      da.qkvg = w.qkvg; da.S = S_qkvg; da.B = x.B; da.dm = dm;
      da.s_q = bw.s_q; da.s_k = bw.s_k;
      da.rope = w.rope + (full ? (size_t)half * 2 : 0);
      da.q_scale = q_scale; da.window = full ? 0 : dm.window;
      da.kv = kv; da.g = geo; da.a_out = w.a; da.err = m->d_status;
      da.row_loops = x.row_loops; da.loop_t = t;
      const double nk = full ? x.n_ctx0 + 1.0
                             : std::min(x.n_ctx0 + 1.0, (double)dm.window);
      if (gemv && x.B * dm.Hkv * nk * dm.hd * 4.0 < kL2pfMaxKvBytes)
        set_l2_prefetch(m, bw, da.l2pf);
      Prof p(m, x.st, "attn_decode",
             x.B * (dm.Hkv * nk * dm.hd * 4.0 + S_qkvg * dm.rows_qkvg * 4.0),
             4.0 * x.B * dm.Hq * nk * dm.hd);
      launch_attn_decode(da, &x.c->kv_maps[2 * slot_index(x.c, i, t)], x.st);
    } else {
      AttnArgs aa{};
      aa.q = w.qb; aa.gate = w.gate; aa.B = x.B; aa.T = x.T; aa.dm = dm;
      aa.window = full ? 0 : dm.window; aa.kv = kv; aa.g = geo;
      aa.a_out = w.a; aa.err = m->d_status;
      double vis = 0;
      for (int t = 0; t < x.T; ++t) {
        const double q = x.n_ctx0 + t + 1.0;
        vis += full ? q : std::min(q, (double)dm.window);
      }
      const double lo = full ? 0 : std::max(0, x.n_ctx0 - dm.window + 1);
      const double keys = x.n_ctx0 + x.T - lo;
      Prof p(m, x.st, "attn_prefill",
             x.B * (dm.Hkv * keys * dm.hd * 4.0) + x.M * dm.qdim * 10.0,
             4.0 * x.B * dm.Hq * vis * dm.hd);
      launch_attn_prefill_tc(aa, &x.c->pf_maps[4 * slot_index(x.c, i, t)], x.st);
    }
    int S_o = 1;
    if (gemv) {
      GemvArgs g{};
      g.W = bw.w_o; g.K = dm.qdim; g.n_items = dm.d; g.B = x.B; g.epi = EPI_F32;
      g.out = w.h;
      g.pro = PRO_BF16; g.xin = w.a; g.xin_stride = dm.qdim;
      S_o = gemv_run(m, g, x.st, "gemv_o", &bw.m_o);
    } else {
      const float* osc = nullptr;
      const bf16* Wo = gemm_weight(m, bw.m_o, dm.d, dm.qdim, w.wdq, x.st, &osc);
      S_o = gemm_run(m, w.a, dm.qdim, Wo, w.h, dm.d, x.M, dm.d, dm.qdim,
                     nullptr, x.st, "gemm_o", slabs, osc);
    }

    // ---- MLP sublayer ---------------------------------------------------
    if (gemv) {
      GemvArgs g{};
      g.W = bw.w_gu; g.K = dm.d; g.n_items = dm.F; g.B = x.B;
      g.epi = EPI_SWIGLU; g.pair_off = dm.F; g.S = 1; g.out_bf = w.mact;
      g.pro = PRO_UPDATE; g.s_in = cur; g.h_in = w.h; g.h_S = S_o;
      g.alpha = bw.alpha_a; g.s_out = other; g.reinject = RJ_NONE; g.x_buf = w.x;
      g.row_loops = x.row_loops; g.upd_loop = t;
      std::swap(cur, other);
      gemv_run(m, g, x.st, "gemv_gateup", &bw.m_gu);
      GemvArgs g2{};
      g2.W = bw.w_down; g2.K = dm.F; g2.n_items = dm.d; g2.B = x.B;
      g2.epi = EPI_F32; g2.out = w.h;
      g2.pro = PRO_BF16; g2.xin = w.mact; g2.xin_stride = dm.F;
      prev_S = gemv_run(m, g2, x.st, "gemv_down", &bw.m_down);
    } else {
      {
        Prof p(m, x.st, "update_rows", (double)x.M * dm.d * 14, 0);
        launch_update_rows(cur, w.h, bw.alpha_a, other, w.s_bf, w.x, RJ_NONE,
                           x.M, dm.d, x.st, S_o, x.row_loops, x.T, t, 0);
      }
      std::swap(cur, other);
      {
        const float* osc = nullptr;
        const bf16* Wgu = gemm_weight(m, bw.m_gu, 2L * dm.F, dm.d, w.wdq, x.st,
                                      &osc);
        Prof p(m, x.st, "gemm_gateup",
               (double)x.M * dm.d * 2 + 2.0 * dm.F * dm.d * 2 +
                   (double)x.M * dm.F * 2,
               2.0 * x.M * 2.0 * dm.F * dm.d);
        launch_gemm_swiglu(w.s_bf, dm.d, Wgu, w.mact, dm.F, x.M, dm.F, dm.d,
                           x.st, osc);
      }
      const float* osc = nullptr;
      const bf16* Wd = gemm_weight(m, bw.m_down, dm.d, dm.F, w.wdq, x.st, &osc);
      prev_S = gemm_run(m, w.mact, dm.F, Wd, w.h, dm.d, x.M, dm.d, dm.F,
                        nullptr, x.st, "gemm_down", slabs, osc);
    }
    prev_alpha = bw.alpha_m;
    prev_t = t;
  }

  // ---- final update and LM head ------------------------------------------
  if (gemv) {
    GemvArgs g{};
    g.W = m->lm_head; g.K = dm.d; g.n_items = dm.V; g.B = x.B; g.S = 1;
    g.epi = EPI_LMHEAD; g.pro = PRO_UPDATE; g.s_in = cur; g.h_in = w.h;
    g.h_S = prev_S; g.alpha = prev_alpha; g.s_out = w.sfin;
    g.reinject = RJ_NONE; g.x_buf = w.x;
    g.row_loops = x.row_loops; g.upd_loop = prev_t;
    g.out = x.logits; g.out_stride = dm.V; g.col_scale = m->s_z;
    g.amax_val = w.amax_val; g.amax_idx = w.amax_idx;
    const int grid = gemv_grid(g, m->num_sms);
    gemv_run(m, g, x.st, "gemv_lmhead");
    if (x.argmax) {
      Prof p(m, x.st, "argmax", x.B * grid * 8.0, 0);
      launch_argmax_partials(w.amax_val, w.amax_idx, x.B, grid, x.argmax,
                             x.c->d_nctx, x.T, x.st);
      return;                  // the argmax kernel advanced the cache length
    }
  } else {
    {
      Prof p(m, x.st, "update_rows", (double)x.M * dm.d * 14, 0);
      launch_update_rows(cur, w.h, prev_alpha, w.sfin, w.s_bf, w.x, RJ_NONE,
                         x.M, dm.d, x.st, prev_S, x.row_loops, x.T, prev_t, 0);
    }
    if (x.logits_all) {
      gemm_run(m, w.s_bf, dm.d, m->lm_head, x.logits, dm.V, x.M, dm.V, dm.d,
               m->s_z, x.st, "gemm_lmhead");
      if (x.argmax) {
        Prof p(m, x.st, "argmax", (double)x.M * dm.V * 4, 0);
        launch_argmax_rows(x.logits, x.M, dm.V, x.argmax, x.st);
      }
    } else if (x.B > 8) {
      // last token of every sequence (rows b*T + T-1, stride T*d) through
      // the tensor-core GEMM: the 671 MB head is read once, not B/8 times
      float* lg = x.logits ? x.logits : w.lg;
      gemm_run(m, w.s_bf + (size_t)(x.T - 1) * dm.d, x.T * dm.d, m->lm_head, lg,
               dm.V, x.B, dm.V, dm.d, m->s_z, x.st, "gemm_lmhead");
      if (x.argmax) {
        Prof p(m, x.st, "argmax", (double)x.B * dm.V * 4, 0);
        launch_argmax_rows(lg, x.B, dm.V, x.argmax, x.st);
      }
    } else {
      for (int b0 = 0; b0 < x.B; b0 += 8) {
        GemvArgs g{};
        g.W = m->lm_head; g.K = dm.d; g.n_items = dm.V; g.S = 1;
        g.B = std::min(8, x.B - b0); g.epi = EPI_LMHEAD; g.pro = PRO_BF16;
        g.xin = w.s_bf + ((size_t)b0 * x.T + x.T - 1) * dm.d;
        g.xin_stride = x.T * dm.d;
        g.out = x.logits ? x.logits + (size_t)b0 * dm.V : nullptr;
        g.out_stride = dm.V; g.col_scale = m->s_z;
        g.amax_val = w.amax_val; g.amax_idx = w.amax_idx;
        const int grid = gemv_grid(g, m->num_sms);
        gemv_run(m, g, x.st, "gemv_lmhead");
        if (x.argmax) {
          Prof p(m, x.st, "argmax", g.B * grid * 8.0, 0);
          launch_argmax_partials(w.amax_val, w.amax_idx, g.B, grid,
                                 x.argmax + b0, nullptr, 0, x.st);
        }
      }
    }
  }
  Prof p(m, x.st, "advance", 8, 0);
  launch_advance(x.c->d_nctx, x.T, x.st);
}

// run_call flags: replay the call from a CUDA graph once its launch plan
// has been seen with the same pointers and shape (calls of up to kMaxGraphT
// tokens); a step of self-speculative decoding (loop counts other than the
// one a per_loop cache is bound to are allowed: the draft runs fewer loops
// than the verifier, whose pass rewrites every slot of the drafted
// positions).
constexpr int kCallGraph = 1, kCallSpec = 2;
constexpr int kMaxGraphT = 16;

int run_call(dory_model* m, dory_cache* c, const int32_t* tokens, int B,
             int T, int n_loops, int kv_mode, int logits_all, float* logits,
             int32_t* argmax, void* ws, int64_t ws_bytes, void* stream,
             int flags, const int* row_loops = nullptr) {
  const bool graphs_ok = (flags & kCallGraph) && T <= kMaxGraphT;
  const bool spec = (flags & kCallSpec) != 0;
  if (!m || !c || c->m != m || !tokens || !ws) return DORY_ERR_ARG;
  if (B != c->B || T < 1 || T > c->max_chunk || n_loops < 1) return DORY_ERR_ARG;
  if (logits_all && !logits) return DORY_ERR_ARG;
  if ((uintptr_t)ws & 255) return DORY_ERR_ARG;
  if (kv_mode != c->kv_mode) return DORY_ERR_CACHE;
  if (kv_mode == DORY_KV_PER_LOOP &&
      (n_loops > c->max_loops ||
       (!spec && c->loops_bound && c->loops_bound != n_loops)))
    return DORY_ERR_CACHE;
  if ((int64_t)c->n_ctx + T > c->max_ctx) return DORY_ERR_CACHE;
  const WS w = ws_layout(m, B, T, (char*)ws);
  if ((int64_t)w.total > ws_bytes) return DORY_ERR_WORKSPACE;
  CallCtx x{m, c, w, B, T, B * T, n_loops, logits_all, c->n_ctx, tokens,
            logits, argmax, (cudaStream_t)stream, row_loops};
  cudaGetLastError();   // clear stale errors from earlier, unrelated calls
  take_host_failure();

  bool done = false;
  if (graphs_ok && m->use_graphs && !m->prof) {
    const GraphKey key(B, n_loops + 256 * T + (logits_all << 24), tokens,
                       logits, argmax, ws, row_loops, c);
    if (m->graphs.size() > 64 && !m->graphs.count(key)) {
      for (auto& kv : m->graphs)
        if (kv.second.exec) cudaGraphExecDestroy(kv.second.exec);
      m->graphs.clear();
    }
    GraphEntry& ge = m->graphs[key];
    if (!ge.exec && ge.seen >= 1) {
      if (!m->cap_stream &&
          cudaStreamCreateWithFlags(&m->cap_stream, cudaStreamNonBlocking) !=
              cudaSuccess)
        return DORY_ERR_CUDA;
      CallCtx cx = x;
      cx.st = m->cap_stream;
      cudaGraph_t graph = nullptr;
      if (cudaStreamBeginCapture(m->cap_stream,
                                 cudaStreamCaptureModeThreadLocal) ==
          cudaSuccess) {
        enqueue_forward(cx);
        const cudaError_t e1 = cudaStreamEndCapture(m->cap_stream, &graph);
        // a launcher that enqueued nothing leaves an incomplete graph
        const bool partial = take_host_failure();
        if (e1 == cudaSuccess && graph && !partial &&
            cudaGraphInstantiate(&ge.exec, graph, 0) != cudaSuccess)
          ge.exec = nullptr;
        if (graph) cudaGraphDestroy(graph);
      }
      cudaGetLastError();
      if (!ge.exec) ge.seen = -1000000;   // never try this key again
    }
    if (ge.exec) {
      if (cudaGraphLaunch(ge.exec, x.st) != cudaSuccess) return DORY_ERR_CUDA;
      done = true;
    } else {
      ge.seen++;
    }
  }
  if (!done) enqueue_forward(x);
  if (take_host_failure() | (cudaGetLastError() != cudaSuccess))
    return DORY_ERR_CUDA;
  c->n_ctx += T;
  if (kv_mode == DORY_KV_PER_LOOP && !c->loops_bound && !spec)
    c->loops_bound = n_loops;
  return DORY_OK;
}

}  // namespace

extern "C" {

int dory_prefill(dory_model* m, dory_cache* c, const int32_t* d_tokens, int B,
                 int T, int n_loops, int kv_mode, int logits_all,
                 float* d_logits, int32_t* d_argmax, void* d_workspace,
                 int64_t ws_bytes, void* stream) {
  return run_call(m, c, d_tokens, B, T, n_loops, kv_mode, logits_all ? 1 : 0,
                  d_logits, d_argmax, d_workspace, ws_bytes, stream, 0);
}

int dory_decode_step(dory_model* m, dory_cache* c, const int32_t* d_tokens,
                     int B, int n_loops, int kv_mode, float* d_logits,
                     int32_t* d_argmax, void* d_workspace, int64_t ws_bytes,
                     void* stream) {
  return run_call(m, c, d_tokens, B, 1, n_loops, kv_mode, 0, d_logits,
                  d_argmax, d_workspace, ws_bytes, stream, kCallGraph);
}

}  // extern "C"

namespace {

// Self-speculative decoding scratch at the head of the caller's workspace:
// draft tokens step-major [gamma+1][B] and row-major [B][gamma+1], the
// verifier's picks [B][gamma+1] and logits [B][gamma+1][V], per-row
// accepted counts, the emitted count.  The forward-pass workspace follows.
struct SpecWS {
  int *steps, *rows, *target, *r, *n_out;
  float* logits;
  size_t total;
};

SpecWS spec_layout(const dory_model* m, int B, int gamma, char* base) {
  const size_t G1 = (size_t)gamma + 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base ? base + off : nullptr;
    off += align256(bytes);
    return p;
  };
  SpecWS w;
  w.steps = (int*)take(G1 * B * 4);
  w.rows = (int*)take(G1 * B * 4);
  w.target = (int*)take(G1 * B * 4);
  w.r = (int*)take((size_t)B * 4);
  w.n_out = (int*)take(4);
  w.logits = (float*)take(G1 * B * m->dm.V * 4);
  w.total = off;
  return w;
}

}  // namespace

extern "C" {

int dory_spec_workspace_bytes(const dory_model* m, int B, int gamma,
                              int64_t* bytes) {
  if (!m || !bytes || B < 1 || gamma < 1 || gamma > 15) return DORY_ERR_ARG;
  int64_t fw = 0;
  const int rc = dory_workspace_bytes(m, B, gamma + 1, &fw);
  if (rc) return rc;
  *bytes = (int64_t)spec_layout(m, B, gamma, nullptr).total + fw;
  return DORY_OK;
}

int dory_spec_decode_step(dory_model* m, dory_cache* c, const int32_t* d_last,
                          int B, int gamma, int k_draft, int k_verify,
                          float temperature, const float* d_uniform,
                          int32_t* d_tokens_out, int* n_out,
                          void* d_workspace, int64_t ws_bytes, void* stream) {
  if (!m || !c || c->m != m || !d_last || !d_tokens_out || !n_out ||
      !d_workspace || B != c->B || gamma < 1 || gamma > 15 || k_draft < 1 ||
      k_verify < k_draft || !(temperature >= 0.f) ||
      (temperature > 0.f && !d_uniform) || ((uintptr_t)d_workspace & 255))
    return DORY_ERR_ARG;
  *n_out = 0;
  if (m->wfmt != DORY_W_BF16) return DORY_ERR_UNSUPPORTED;
  if (gamma + 1 > c->max_chunk) return DORY_ERR_ARG;
  const int n0 = c->n_ctx;
  if ((int64_t)n0 + gamma + 1 > c->max_ctx) return DORY_ERR_CACHE;
  // per_loop only: there a multi-token pass computes what one-token steps
  // compute, so the verifier's picks are those of plain decoding (in
  // last_loop mode a chunk's tokens read same-loop entries of each other)
  if (c->kv_mode != DORY_KV_PER_LOOP || k_verify > c->max_loops ||
      (c->loops_bound && c->loops_bound != k_verify))
    return DORY_ERR_CACHE;
  const SpecWS sw = spec_layout(m, B, gamma, (char*)d_workspace);
  if ((int64_t)sw.total >= ws_bytes) return DORY_ERR_WORKSPACE;
  char* fws = (char*)d_workspace + sw.total;
  const int64_t fws_bytes = ws_bytes - (int64_t)sw.total;
  const cudaStream_t st = (cudaStream_t)stream;
  const int G1 = gamma + 1;
  cudaGetLastError();
  if (cudaMemcpyAsync(sw.steps, d_last, (size_t)B * 4, cudaMemcpyDeviceToDevice,
                      st) != cudaSuccess)
    return DORY_ERR_CUDA;
  // draft: gamma greedy decode steps at k_draft loops, each token written
  // straight into the input of the next
  for (int j = 0; j < gamma; ++j) {
    const int rc = run_call(m, c, sw.steps + (size_t)j * B, B, 1, k_draft,
                            c->kv_mode, 0, nullptr, sw.steps + (size_t)(j + 1) * B,
                            fws, fws_bytes, stream, kCallGraph | kCallSpec);
    if (rc) {
      c->n_ctx = n0;
      launch_set_nctx(c->d_nctx, n0, st);
      return rc;
    }
  }
  // verify: the last accepted token and the gamma drafts at k_verify loops
  // in one multi-token pass from position n0; every slot of those positions
  // is rewritten before it is read
  c->n_ctx = n0;
  launch_set_nctx(c->d_nctx, n0, st);
  launch_spec_transpose(sw.steps, sw.rows, B, G1, st);
  int rc = run_call(m, c, sw.rows, B, G1, k_verify, c->kv_mode, 1, sw.logits,
                    sw.target, fws, fws_bytes, stream, kCallGraph | kCallSpec);
  if (rc) {
    c->n_ctx = n0;
    launch_set_nctx(c->d_nctx, n0, st);
    return rc;
  }
  SpecArgs a{};
  a.draft = sw.rows; a.target = sw.target; a.logits = sw.logits;
  a.uniform = d_uniform; a.B = B; a.gamma = gamma; a.V = m->dm.V;
  a.inv_temp = temperature > 0.f ? 1.f / temperature : 0.f;
  a.r = sw.r; a.out = d_tokens_out; a.n_out = sw.n_out; a.n_ctx = c->d_nctx;
  a.n0 = n0;
  launch_spec_accept(a, st);
  int n = 0;
  if (cudaGetLastError() != cudaSuccess ||
      cudaMemcpyAsync(&n, sw.n_out, 4, cudaMemcpyDeviceToHost, st) !=
          cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess || n < 1 || n > G1) {
    c->n_ctx = n0;
    return DORY_ERR_CUDA;
  }
  c->n_ctx = n0 + n;
  if (!c->loops_bound) c->loops_bound = k_verify;
  *n_out = n;
  return DORY_OK;
}

int dory_debug_spec_accept(const int32_t* d_draft, const int32_t* d_target,
                           const float* d_logits, const float* d_uniform,
                           int B, int gamma, int V, float temperature,
                           int32_t* d_tokens_out, int32_t* d_scratch,
                           void* stream) {
  if (!d_draft || !d_target || !d_tokens_out || !d_scratch || B < 1 ||
      gamma < 1 || V < 2 || !(temperature >= 0.f) ||
      (temperature > 0.f && (!d_uniform || !d_logits)))
    return DORY_ERR_ARG;
  SpecArgs a{};
  a.draft = d_draft; a.target = d_target; a.logits = d_logits;
  a.uniform = d_uniform; a.B = B; a.gamma = gamma; a.V = V;
  a.inv_temp = temperature > 0.f ? 1.f / temperature : 0.f;
  a.r = d_scratch + 2; a.out = d_tokens_out; a.n_out = d_scratch;
  a.n_ctx = d_scratch + 1; a.n0 = 0;
  cudaGetLastError();
  launch_spec_accept(a, (cudaStream_t)stream);
  return cuda_rc(cudaGetLastError());
}

int dory_prefill_mixed(dory_model* m, dory_cache* c, const int32_t* d_tokens,
                       int B, int T, const int32_t* d_row_loops, int max_loops,
                       int kv_mode, int logits_all, float* d_logits,
                       int32_t* d_argmax, void* d_workspace, int64_t ws_bytes,
                       void* stream) {
  if (!d_row_loops) return DORY_ERR_ARG;
  return run_call(m, c, d_tokens, B, T, max_loops, kv_mode, logits_all ? 1 : 0,
                  d_logits, d_argmax, d_workspace, ws_bytes, stream, 0,
                  d_row_loops);
}

int dory_decode_step_mixed(dory_model* m, dory_cache* c,
                           const int32_t* d_tokens, int B,
                           const int32_t* d_row_loops, int max_loops,
                           int kv_mode, float* d_logits, int32_t* d_argmax,
                           void* d_workspace, int64_t ws_bytes, void* stream) {
  if (!d_row_loops) return DORY_ERR_ARG;
  return run_call(m, c, d_tokens, B, 1, max_loops, kv_mode, 0, d_logits,
                  d_argmax, d_workspace, ws_bytes, stream, kCallGraph,
                  d_row_loops);
}

int dory_copy_state(const dory_model* m, const void* d_workspace, int B,
                    int T, int logits_all, float* d_out, void* stream) {
  if (!m || !d_workspace || !d_out || B < 1 || T < 1) return DORY_ERR_ARG;
  const WS w = ws_layout(m, B, T, (char*)d_workspace);
  const size_t row = (size_t)m->dm.d * sizeof(float);
  cudaError_t e;
  if (use_gemv(B, T) || logits_all)
    e = cudaMemcpyAsync(d_out, w.sfin, row * B * (logits_all ? T : 1),
                        cudaMemcpyDeviceToDevice, (cudaStream_t)stream);
  else
    e = cudaMemcpy2DAsync(d_out, row, w.sfin + (size_t)(T - 1) * m->dm.d,
                          row * T, row, B, cudaMemcpyDeviceToDevice,
                          (cudaStream_t)stream);
  return cuda_rc(e);
}

int dory_sync_status(dory_model* m, void* stream) {
  if (!m) return DORY_ERR_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess)
    return DORY_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_dory_status, sizeof(int)) != cudaSuccess)
    return DORY_ERR_CUDA;
  if (v) {
    const int zero = 0;
    cudaMemcpyToSymbol(g_dory_status, &zero, sizeof(int));
  }
  if (v & ERRBIT_TIMEOUT) return DORY_ERR_TIMEOUT;
  if (v) return DORY_ERR_DEVICE;
  return DORY_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free decode step (dory_decode_step_static).  Its workspace is a
// file-scope device array; host code reaches it only through the address
// that cudaGetSymbolAddress returns for the current device (the symbol's
// name in host code is a host-side stand-in, not a device address).
static __device__ __align__(256) unsigned char g_static_ws[DORY_STATIC_WS_BYTES];

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_static_ws_mu;
void* g_static_ws_addr[kMaxDevices];

// Device address of this device's copy of g_static_ws, looked up once per
// device with that device current.
int static_ws_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return DORY_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DORY_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_ws_mu);
  if (!g_static_ws_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p)
      return DORY_ERR_CUDA;
    g_static_ws_addr[dev] = p;
  }
  *out = g_static_ws_addr[dev];
  return DORY_OK;
}

}  // namespace

extern "C" int dory_decode_step_static(dory_model* m, dory_cache* c,
                                       const int32_t* d_tokens, int B,
                                       int n_loops, int kv_mode,
                                       float* d_logits, int32_t* d_argmax,
                                       void* stream) {
  if (!m || !c || B < 1) return DORY_ERR_ARG;
  int64_t need = 0;
  const int rc0 = dory_workspace_bytes(m, B, 1, &need);
  if (rc0) return rc0;
  if (need > (int64_t)DORY_STATIC_WS_BYTES) return DORY_ERR_WORKSPACE;
  void* ws = nullptr;
  const int rc = static_ws_address(&ws);
  if (rc) return rc;
  // flags 0: the kernels are launched directly, never via a graph.
  return run_call(m, c, d_tokens, B, 1, n_loops, kv_mode, 0, d_logits,
                  d_argmax, ws, (int64_t)DORY_STATIC_WS_BYTES, stream, 0);
}

// A bounded wait that runs out on purpose: one thread waits on an mbarrier
// that nothing arrives on, gives up after `polls` polls and records
// ERRBIT_TIMEOUT, exactly as the streaming kernels do when a copy or a peer
// stalls.  No copy is in flight and no tensor memory is held.
__global__ void bounded_wait_kernel(int polls, int* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (!mbar_wait(&bar, 0, polls)) atomicOr(err, ERRBIT_TIMEOUT);
  }
}

extern "C" int dory_debug_bounded_wait(dory_model* m, int polls,
                                       void* stream) {
  if (!m || polls < 1 || polls > (1 << 20)) return DORY_ERR_ARG;
  cudaGetLastError();
  bounded_wait_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(polls, m->d_status);
  return cuda_rc(cudaGetLastError());
}

extern "C" int dory_debug_gemm_bf16(const void* d_A, int lda, const void* d_W,
                                    float* d_C, int M, int N, int K,
                                    void* stream) {
  if (!d_A || !d_W || !d_C || M < 1 || N < 1 || K < 64 || K % 64 ||
      lda < K || lda % 8)
    return DORY_ERR_ARG;
  cudaGetLastError();
  take_host_failure();
  launch_gemm_bf16((const bf16*)d_A, lda, (const bf16*)d_W, d_C, N, M, N, K,
                   nullptr, (cudaStream_t)stream);
  if (take_host_failure()) return DORY_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? DORY_OK : DORY_ERR_CUDA;
}

extern "C" int dory_debug_gemm_bf16_split(const void* d_A, int lda,
                                          const void* d_W, float* d_C, int M,
                                          int N, int K, int max_splits,
                                          int* n_partials, void* stream) {
  if (!d_A || !d_W || !d_C || !n_partials || M < 1 || N < 1 || K < 64 ||
      K % 64 || lda < K || lda % 8 || max_splits < 1)
    return DORY_ERR_ARG;
  cudaGetLastError();
  take_host_failure();
  *n_partials = launch_gemm_bf16((const bf16*)d_A, lda, (const bf16*)d_W, d_C,
                                 N, M, N, K, nullptr, (cudaStream_t)stream,
                                 max_splits, (long)M * N);
  if (take_host_failure()) {
    *n_partials = 0;
    return DORY_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? DORY_OK : DORY_ERR_CUDA;
}

extern "C" int dory_cache_fill_synthetic(dory_model* m, dory_cache* c,
                                         int n_ctx, uint64_t seed,
                                         void* stream) {
  if (!m || !c || c->m != m || n_ctx < 0 || n_ctx > c->max_ctx)
    return DORY_ERR_ARG;
  const Dims& dm = m->dm;
  const cudaStream_t st = (cudaStream_t)stream;
  const CacheGeo geo{c->d_nctx, c->d_block_table, c->pages_per_seq,
                     c->max_ctx};
  const float ck = (float)std::sqrt(3.0 / dm.hd);
  const float cv = (float)std::sqrt(3.0 / dm.d);
  cudaGetLastError();
  for (int i = 0; i < m->nblk; ++i) {
    const int ns = slots_of(m, i, c->kv_mode, c->max_loops);
    for (int s2 = 0; s2 < ns; ++s2) {
      const KVSlot& kv = c->slots[c->slot_base[i] + s2];
      // the generator's slot index: loop t (1-based) of a per_loop
      // recurrent block, 0 for every single-slot block
      const int gslot = (ns > 1 || (is_rec(m, i) &&
                                     c->kv_mode == DORY_KV_PER_LOOP))
                            ? s2 + 1 : 0;
      const int lo = kv.ring ? std::max(0, n_ctx - kv.cap) : 0;
      launch_fill_kv(kv, geo, c->B, dm.Hkv, dm.hd, lo, n_ctx, i, gslot, seed,
                     ck, cv, st);
    }
  }
  launch_set_nctx(c->d_nctx, n_ctx, st);
  if (cudaGetLastError() != cudaSuccess) return DORY_ERR_CUDA;
  c->n_ctx = n_ctx;
  c->loops_bound = 0;
  return DORY_OK;
}

namespace {

// Block projection `tensor` ("blk<i>.<w>") of a model: its matrix and shape.
bool find_proj(const dory_model* m, const char* tensor, const QMat** q,
               long* N, long* K) {
  if (!tensor) return false;
  const std::string n = tensor;
  if (n.compare(0, 3, "blk") != 0) return false;
  const size_t dot = n.find('.');
  if (dot == std::string::npos || dot == 3) return false;
  for (size_t c = 3; c < dot; ++c)
    if (n[c] < '0' || n[c] > '9') return false;
  const int i = atoi(n.substr(3, dot - 3).c_str());
  if (i < 0 || i >= m->nblk) return false;
  const std::string leaf = n.substr(dot + 1);
  const BlockW& b = m->blk[i];
  const Dims& dm = m->dm;
  if (leaf == "w_qkvg") { *q = &b.m_qkvg; *N = dm.rows_qkvg; *K = dm.d; }
  else if (leaf == "w_o") { *q = &b.m_o; *N = dm.d; *K = dm.qdim; }
  else if (leaf == "w_gu") { *q = &b.m_gu; *N = 2L * dm.F; *K = dm.d; }
  else if (leaf == "w_down") { *q = &b.m_down; *N = dm.d; *K = dm.F; }
  else return false;
  return true;
}

}  // namespace

extern "C" int dory_debug_gemv(const dory_model* m, const char* tensor,
                               const void* d_x, int B, float* d_out,
                               int max_partials, int* n_partials,
                               void* stream) {
  if (!m || !d_x || !d_out || !n_partials || B < 1 || B > 8 ||
      max_partials < 1 || ((uintptr_t)d_x & 15))
    return DORY_ERR_ARG;
  *n_partials = 0;
  const QMat* q = nullptr;
  long N = 0, K = 0;
  if (!find_proj(m, tensor, &q, &N, &K)) return DORY_ERR_ARG;
  GemvArgs g{};
  g.W = q->w;
  g.fmt = WF_BF16;
  if (!q->w) {
    g.fmt = m->wfmt == DORY_W_MXFP8 ? WF_MXFP8 : WF_NVFP4;
    g.Wq = q->q;
    g.Ws = q->s;
    g.Wt = q->t;
  }
  g.K = (int)K;
  g.n_items = (int)N;
  g.B = B;
  g.epi = EPI_F32;
  g.pro = PRO_BF16;
  g.xin = (const bf16*)d_x;
  g.xin_stride = (int)K;
  g.out = d_out;
  g.err = m->d_status;
  g.S = gemv_splits(g);
  if (g.S > max_partials) return DORY_ERR_ARG;
  cudaGetLastError();
  launch_gemv(g, gemv_grid(g, m->num_sms), (cudaStream_t)stream);
  if (cudaGetLastError() != cudaSuccess) return DORY_ERR_CUDA;
  *n_partials = g.S;
  return DORY_OK;
}

extern "C" int dory_cache_copy_prefix(dory_model* m, dory_cache* dst,
                                      const dory_cache* src, int src_b,
                                      int n_tokens, void* stream) {
  if (!m || !dst || !src || dst == src || dst->m != m || src->m != m ||
      src_b < 0 || src_b >= src->B || n_tokens < 0)
    return DORY_ERR_ARG;
  if (dst->kv_mode != src->kv_mode || n_tokens > src->n_ctx ||
      n_tokens > dst->max_ctx)
    return DORY_ERR_CACHE;
  // the loops the source's per_loop slots hold
  int loops = 1;
  if (src->kv_mode == DORY_KV_PER_LOOP) {
    loops = src->loops_bound;
    if (n_tokens > 0 && loops == 0) return DORY_ERR_CACHE;
    if (loops > dst->max_loops) return DORY_ERR_CACHE;
  }
  const Dims& dm = m->dm;
  // a later query at position n_tokens sees sliding-window keys from
  // n_tokens - W + 1 on; the source ring must still hold them
  const int sw_lo = std::max(0, n_tokens - dm.window + 1);
  if (n_tokens > 0 && src->n_ctx - src->swa_cap > sw_lo) return DORY_ERR_CACHE;
  const cudaStream_t st = (cudaStream_t)stream;
  const CacheGeo gs{src->d_nctx, src->d_block_table, src->pages_per_seq,
                    src->max_ctx};
  const CacheGeo gd{dst->d_nctx, dst->d_block_table, dst->pages_per_seq,
                    dst->max_ctx};
  cudaGetLastError();
  for (int i = 0; i < m->nblk; ++i) {
    const bool per_loop = is_rec(m, i) && src->kv_mode == DORY_KV_PER_LOOP;
    const int ns = per_loop ? loops : 1;
    for (int t = 0; t < ns; ++t) {
      const KVSlot& a = src->slots[src->slot_base[i] + t];
      const KVSlot& b = dst->slots[dst->slot_base[i] + t];
      const int lo = a.ring ? sw_lo : 0;
      launch_copy_prefix(a, gs, src_b, b, gd, dst->B, dm.Hkv, dm.hd, lo,
                         n_tokens, st);
    }
  }
  launch_set_nctx(dst->d_nctx, n_tokens, st);
  if (cudaGetLastError() != cudaSuccess) return DORY_ERR_CUDA;
  dst->n_ctx = n_tokens;
  dst->loops_bound = src->kv_mode == DORY_KV_PER_LOOP && n_tokens > 0
                         ? loops : 0;
  return DORY_OK;
}

extern "C" int dory_debug_dequant(const dory_model* m, const char* tensor,
                                  int row0, int nrows, float* d_out,
                                  void* stream) {
  if (!m || !tensor || !d_out || row0 < 0 || nrows < 1) return DORY_ERR_ARG;
  if (m->wfmt == DORY_W_BF16) return DORY_ERR_UNSUPPORTED;
  const QMat* q = nullptr;
  long N = 0, K = 0;
  if (!find_proj(m, tensor, &q, &N, &K)) return DORY_ERR_ARG;
  if ((long)row0 + nrows > N) return DORY_ERR_ARG;
  cudaGetLastError();
  launch_dequant_rows(m->wfmt == DORY_W_MXFP8 ? WF_MXFP8 : WF_NVFP4, q->q, q->s,
                      (int)K, row0, nrows, d_out, (cudaStream_t)stream);
  return cudaGetLastError() == cudaSuccess ? DORY_OK : DORY_ERR_CUDA;
}
