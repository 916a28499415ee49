// C ABI of the decode-step library: host-side validation, workspace layout, launches.
// Every entry point validates synchronously, launches asynchronously on the caller's
// stream, and never synchronizes or allocates.
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "internal.h"

namespace dsv4 {

int sm_count() {
  static std::mutex mu;
  static std::vector<int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, 0);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {
std::atomic<uint64_t> g_launches{0};
}

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

}  // namespace dsv4

using namespace dsv4;

namespace {

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_dtype(dsv4_dtype d) { return d == DSV4_F32 || d == DSV4_BF16 || d == DSV4_FP8E4M3; }
// caches may also hold fp4 rows (indexer keys)
bool valid_cache_dtype(dsv4_dtype d) { return valid_dtype(d) || d == DSV4_FP4E2M1; }
size_t dsize(dsv4_dtype d) { return d == DSV4_F32 ? 4 : (d == DSV4_BF16 ? 2 : 1); }
size_t row_bytes(dsv4_dtype d, int dim) { return d == DSV4_FP4E2M1 ? static_cast<size_t>(dim) / 2 : dim * dsize(d); }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

dsv4_status to_status(cudaError_t e) {
  if (e == cudaSuccess) return DSV4_OK;
  cudaGetLastError();  // clear a sticky launch-configuration error
  return DSV4_ERR_CUDA;
}

bool valid_rope(const dsv4_rope &r, int dim) {
  return r.rope_dims >= 0 && r.rope_dims % 2 == 0 && r.rope_dims <= dim && (r.rope_dims == 0 || r.rope_base > 0.f);
}

// a paged cache: pointers, dims, alignment
bool valid_cache(const dsv4_paged_cache &c, bool need_scales_if_fp8 = true) {
  if (!c.pages || !c.block_table || c.num_pages <= 0 || c.max_blocks <= 0 || c.dim <= 0) return false;
  if (!pow2(c.m) || c.m > DSV4_PAGE_POSITIONS || !valid_cache_dtype(c.dtype)) return false;
  if (c.dtype == DSV4_FP4E2M1 && c.dim % 2 != 0) return false;
  if (!aligned16(c.pages) || row_bytes(c.dtype, c.dim) % 16 != 0) return false;
  if ((c.dtype == DSV4_FP8E4M3 || c.dtype == DSV4_FP4E2M1) && need_scales_if_fp8 && (!c.scales || !aligned16(c.scales)))
    return false;
  return true;
}

bool valid_ring(const dsv4_window_ring &r) {
  if (!r.rows || r.window <= 0 || r.dim <= 0 || !valid_dtype(r.dtype)) return false;
  if (!aligned16(r.rows) || (r.dim * dsize(r.dtype)) % 16 != 0) return false;
  if (r.dtype == DSV4_FP8E4M3 && !r.scales) return false;
  return true;
}

bool valid_state(const dsv4_compressor_state &s) {
  return s.buf && s.m > 0 && s.dim > 0 && (s.gate_dim == s.dim || s.gate_dim == 1) && aligned16(s.buf);
}

// vector width handled by the pooling kernels: a power of two in [32, 2048]
bool valid_pool_dim(int d) { return pow2(d) && d >= 32 && d <= 2048; }

}  // namespace

namespace {
// the checks of dsv4_compress that do not look at kv, gate and kv_dtype
dsv4_status check_compress_common(const dsv4_compress_args *a) {
  if (a->batch <= 0 || a->batch > 16384 || a->total_tokens < 0) return DSV4_ERR_INVALID_ARG;
  if (!a->cu_seqlens || !a->start_pos || !a->gamma) return DSV4_ERR_INVALID_ARG;
  if (!valid_state(a->state) || !valid_cache(a->cache)) return DSV4_ERR_INVALID_ARG;
  if (a->state.m != a->cache.m || a->state.dim != a->cache.dim) return DSV4_ERR_INVALID_ARG;
  if (!valid_rope(a->rope, a->state.dim) || !(a->eps >= 0.f)) return DSV4_ERR_INVALID_ARG;
  if (!valid_pool_dim(a->state.dim)) return DSV4_ERR_UNSUPPORTED;
  return DSV4_OK;
}

// the projection's own rules (beside those of dsv4_compress); DSV4_OK or the error
dsv4_status check_project(const dsv4_compress_project_args *a) {
  if (!a) return DSV4_ERR_INVALID_ARG;
  const dsv4_status c = check_compress_common(&a->c);
  if (c != DSV4_OK) return c;
  if (a->c.total_tokens > 0 && (!a->hidden || !a->w)) return DSV4_ERR_INVALID_ARG;
  if (!aligned16(a->hidden) || !aligned16(a->w)) return DSV4_ERR_INVALID_ARG;
  if (a->hidden_dim <= 0) return DSV4_ERR_INVALID_ARG;
  if (a->c.state.gate_dim != a->c.state.dim) return DSV4_ERR_UNSUPPORTED;
  if (a->hidden_dim % 64 != 0 || a->c.state.dim % 128 != 0) return DSV4_ERR_UNSUPPORTED;
  return DSV4_OK;
}
}  // namespace

extern "C" {

const char *dsv4_status_string(dsv4_status s) {
  switch (s) {
    case DSV4_OK: return "ok";
    case DSV4_ERR_INVALID_ARG: return "invalid argument";
    case DSV4_ERR_UNSUPPORTED: return "unsupported combination";
    case DSV4_ERR_CUDA: return "CUDA launch error";
    case DSV4_ERR_SCRATCH_LIMIT: return "request exceeds the library's static scratch";
  }
  return "unknown status";
}

int32_t dsv4_abi_version(void) { return DSV4_ABI_VERSION; }

uint64_t dsv4_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

uint64_t dsv4_layer_state_bytes(uint64_t context, int32_t m, int32_t entry_width, int32_t window, int32_t window_width,
                                int32_t bytes_per_value) {
  if (m <= 0 || entry_width < 0 || window < 0 || window_width < 0 || bytes_per_value <= 0) return 0;
  return (context / static_cast<uint64_t>(m)) * static_cast<uint64_t>(entry_width) * bytes_per_value +
         static_cast<uint64_t>(window) * static_cast<uint64_t>(window_width) * bytes_per_value;
}

// ------------------------------------------------------------------------------------
dsv4_status dsv4_compress(const dsv4_compress_args *a, dsv4_stream stream) {
  if (!a) return DSV4_ERR_INVALID_ARG;
  const dsv4_status c = check_compress_common(a);
  if (c != DSV4_OK) return c;
  if (a->total_tokens > 0 && (!a->kv || !a->gate)) return DSV4_ERR_INVALID_ARG;
  if (a->kv_dtype != DSV4_F32 && a->kv_dtype != DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
  if (!aligned16(a->kv) || !aligned16(a->gate)) return DSV4_ERR_INVALID_ARG;
  if (a->total_tokens == 0) return DSV4_OK;
  CompressLaunch p{};
  p.B = a->batch;
  p.total_tokens = a->total_tokens;
  p.kv = a->kv;
  p.gate = a->gate;
  p.kv_dt = a->kv_dtype;
  p.cu_seqlens = a->cu_seqlens;
  p.start_pos = a->start_pos;
  p.gamma = a->gamma;
  p.eps = a->eps;
  p.rope_dims = a->rope.rope_dims;
  p.rope_base = a->rope.rope_base;
  p.state = a->state.buf;
  p.m = a->state.m;
  p.D = a->state.dim;
  p.G = a->state.gate_dim;
  p.pages = a->cache.pages;
  p.scales = a->cache.scales;
  p.block_table = a->cache.block_table;
  p.num_pages = a->cache.num_pages;
  p.max_blocks = a->cache.max_blocks;
  p.cache_dt = a->cache.dtype;
  p.d_status = a->d_status;
  return to_status(launch_compress(p, static_cast<cudaStream_t>(stream)));
}

size_t dsv4_compress_project_workspace_size(const dsv4_compress_project_args *a) {
  if (check_project(a) != DSV4_OK) return 0;
  return 2 * project_out_bytes(a->c.total_tokens, a->c.state.dim) + 256;
}

dsv4_status dsv4_compress_project(const dsv4_compress_project_args *a, void *ws, size_t ws_bytes,
                                  dsv4_stream stream) {
  const dsv4_status c = check_project(a);
  if (c != DSV4_OK) return c;
  if (a->c.total_tokens == 0) return DSV4_OK;
  if (!ws || reinterpret_cast<uintptr_t>(ws) % 256 != 0 || ws_bytes < dsv4_compress_project_workspace_size(a))
    return DSV4_ERR_INVALID_ARG;
  const int T = a->c.total_tokens, D = a->c.state.dim;
  ProjectLaunch pj{};
  pj.hidden = a->hidden;
  pj.w = a->w;
  pj.kv = static_cast<uint16_t *>(ws);
  pj.gate = reinterpret_cast<uint16_t *>(static_cast<char *>(ws) + project_out_bytes(T, D));
  pj.T = T;
  pj.D = D;
  pj.Hd = a->hidden_dim;
  pj.d_status = a->c.d_status;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = launch_project(pj, st);
  if (e != cudaSuccess) return to_status(e);
  dsv4_compress_args cc = a->c;
  cc.kv = pj.kv;
  cc.gate = pj.gate;
  cc.kv_dtype = DSV4_BF16;
  return dsv4_compress(&cc, stream);
}

dsv4_status dsv4_swa_insert(const dsv4_swa_insert_args *a, dsv4_stream stream) {
  if (!a) return DSV4_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->batch > 65535 || a->total_tokens < 0) return DSV4_ERR_INVALID_ARG;
  if (!a->cu_seqlens || !a->start_pos || !a->gamma) return DSV4_ERR_INVALID_ARG;
  if (a->total_tokens > 0 && !a->kv) return DSV4_ERR_INVALID_ARG;
  if (!valid_ring(a->ring) || !valid_rope(a->rope, a->ring.dim) || !(a->eps >= 0.f)) return DSV4_ERR_INVALID_ARG;
  if (a->kv_dtype != DSV4_F32 && a->kv_dtype != DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
  if (a->ring.dim > 2048 || a->ring.dim % 2 != 0 || a->ring.window > 65535) return DSV4_ERR_UNSUPPORTED;
  if (a->total_tokens == 0) return DSV4_OK;
  SwaLaunch p{};
  p.B = a->batch;
  p.total_tokens = a->total_tokens;
  p.kv = a->kv;
  p.kv_dt = a->kv_dtype;
  p.cu_seqlens = a->cu_seqlens;
  p.start_pos = a->start_pos;
  p.gamma = a->gamma;
  p.eps = a->eps;
  p.rope_dims = a->rope.rope_dims;
  p.rope_base = a->rope.rope_base;
  p.rows = a->ring.rows;
  p.scales = a->ring.scales;
  p.W = a->ring.window;
  p.D = a->ring.dim;
  p.ring_dt = a->ring.dtype;
  p.d_status = a->d_status;
  return to_status(launch_swa_insert(p, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------------------------
static dsv4_status indexer_launch_args(const dsv4_indexer_args *a, IndexerLaunch *p) {
  if (!a) return DSV4_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->batch > 65535 || a->heads <= 0 || a->dim <= 0 || a->k <= 0) return DSV4_ERR_INVALID_ARG;
  if (!a->q_idx || !a->w || !a->n_entries || !a->idx) return DSV4_ERR_INVALID_ARG;
  if (!valid_cache(a->keys) || a->keys.dim != a->dim) return DSV4_ERR_INVALID_ARG;
  if (a->q_rope_dims < 0 || a->q_rope_dims % 2 != 0 || a->q_rope_dims > a->dim) return DSV4_ERR_INVALID_ARG;
  if (a->q_rope_dims > 0 && (!a->pos || !(a->rope_base > 0.f))) return DSV4_ERR_INVALID_ARG;
  if (a->q_dtype != DSV4_F32 && a->q_dtype != DSV4_FP8E4M3) return DSV4_ERR_UNSUPPORTED;
  if (a->w_dtype != DSV4_F32 && a->w_dtype != DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
  if (a->keys.dtype == DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
  if (a->q_rope_dims > 0 && a->q_dtype != DSV4_F32) return DSV4_ERR_UNSUPPORTED;
  if (a->k > 2048 || static_cast<int64_t>(a->heads) * a->dim > 8192) return DSV4_ERR_UNSUPPORTED;
  if (!aligned16(a->q_idx)) return DSV4_ERR_INVALID_ARG;
  *p = IndexerLaunch{};
  p->B = a->batch;
  p->H = a->heads;
  p->Dq = a->dim;
  p->k = a->k;
  p->q = a->q_idx;
  p->q_dt = a->q_dtype;
  p->q_scale = a->q_scale;
  p->w = a->w;
  p->w_dt = a->w_dtype;
  p->k_pages = a->keys.pages;
  p->k_scales = a->keys.scales;
  p->block_table = a->keys.block_table;
  p->num_pages = a->keys.num_pages;
  p->max_blocks = a->keys.max_blocks;
  p->m = a->keys.m;
  p->k_dt = a->keys.dtype;
  p->n_entries = a->n_entries;
  p->pos = a->pos;
  p->q_rope_dims = a->q_rope_dims;
  p->rope_base = a->rope_base;
  p->idx = a->idx;
  p->scores = a->scores;
  p->d_status = a->d_status;
  return DSV4_OK;
}

size_t dsv4_indexer_workspace_size(const dsv4_indexer_args *a) {
  IndexerLaunch p;
  if (indexer_launch_args(a, &p) != DSV4_OK) return 0;
  return indexer_workspace_bytes(p);
}

dsv4_status dsv4_indexer_topk(const dsv4_indexer_args *a, void *ws, size_t ws_bytes, dsv4_stream stream) {
  IndexerLaunch p;
  const dsv4_status s = indexer_launch_args(a, &p);
  if (s != DSV4_OK) return s;
  const size_t need = indexer_workspace_bytes(p);
  if (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u)) return DSV4_ERR_INVALID_ARG;
  return to_status(launch_indexer_topk(p, ws, static_cast<cudaStream_t>(stream)));
}

dsv4_status dsv4_indexer_scores(const dsv4_indexer_args *a, float *scores, int64_t scores_ld, dsv4_stream stream) {
  if (!a) return DSV4_ERR_INVALID_ARG;
  dsv4_indexer_args b = *a;
  int32_t dummy_idx = 0;
  if (!b.idx) b.idx = &dummy_idx;  // (the selection's output is not used here)
  IndexerLaunch p;
  const dsv4_status s = indexer_launch_args(&b, &p);
  if (s != DSV4_OK) return s;
  if (!indexer_uses_tensor_cores(p)) return DSV4_ERR_UNSUPPORTED;
  if (!scores || (reinterpret_cast<uintptr_t>(scores) & 15u) || scores_ld < indexer_score_capacity(p) ||
      scores_ld % 4 != 0)
    return DSV4_ERR_INVALID_ARG;
  p.idx = nullptr;
  return to_status(launch_indexer_scores(p, scores, scores_ld, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------------------------
static dsv4_status mqa_launch_args(const dsv4_mqa_args *a, MqaLaunch *p) {
  if (!a) return DSV4_ERR_INVALID_ARG;
  if (a->batch <= 0 || a->batch > 65535 || a->heads <= 0 || a->heads > 65535 || a->dim <= 0)
    return DSV4_ERR_INVALID_ARG;
  if (!a->q || !a->pos || !a->out) return DSV4_ERR_INVALID_ARG;
  if (!valid_cache(a->cache) || !valid_ring(a->ring)) return DSV4_ERR_INVALID_ARG;
  if (a->cache.dim != a->dim || a->ring.dim != a->dim || a->cache.dtype != a->ring.dtype) return DSV4_ERR_INVALID_ARG;
  if (a->cache.dtype == DSV4_FP4E2M1) return DSV4_ERR_UNSUPPORTED;  // fp4 is for indexer keys only
  if (a->idx && a->k <= 0) return DSV4_ERR_INVALID_ARG;
  if (!a->idx && !a->n_entries) return DSV4_ERR_INVALID_ARG;
  if (!valid_rope(a->rope, a->dim)) return DSV4_ERR_INVALID_ARG;
  if (a->q_dtype != DSV4_F32 && a->q_dtype != DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
  if (!valid_dtype(a->out_dtype)) return DSV4_ERR_UNSUPPORTED;
  if (a->out_dtype == DSV4_FP8E4M3 && (!a->out_scales || a->dim % kOutBlock != 0)) return DSV4_ERR_INVALID_ARG;
  if (a->q_norm_gamma && !(a->q_norm_eps >= 0.f)) return DSV4_ERR_INVALID_ARG;
  if (a->dim > 1024 || a->dim % 32 != 0) return DSV4_ERR_UNSUPPORTED;
  if (!aligned16(a->q) || !aligned16(a->out)) return DSV4_ERR_INVALID_ARG;
  *p = MqaLaunch{};
  p->B = a->batch;
  p->H = a->heads;
  p->D = a->dim;
  p->q = a->q;
  p->q_dt = a->q_dtype;
  p->pos = a->pos;
  p->pages = a->cache.pages;
  p->scales = a->cache.scales;
  p->block_table = a->cache.block_table;
  p->num_pages = a->cache.num_pages;
  p->max_blocks = a->cache.max_blocks;
  p->m = a->cache.m;
  p->kv_dt = a->cache.dtype;
  p->n_entries = a->n_entries;
  p->idx = a->idx;
  p->k = a->idx ? a->k : 0;
  p->ring_rows = a->ring.rows;
  p->ring_scales = a->ring.scales;
  p->W = a->ring.window;
  p->softmax_scale = a->softmax_scale;
  p->rope_dims = a->rope.rope_dims;
  p->rope_base = a->rope.rope_base;
  p->out = a->out;
  p->out_dt = a->out_dtype;
  p->lse = a->lse;
  p->d_status = a->d_status;
  p->q_norm_gamma = a->q_norm_gamma;
  p->q_norm_eps = a->q_norm_eps;
  p->out_scales = a->out_scales;
  return DSV4_OK;
}

size_t dsv4_mqa_workspace_size(const dsv4_mqa_args *a) {
  MqaLaunch p;
  if (mqa_launch_args(a, &p) != DSV4_OK) return 0;
  return mqa_workspace_bytes(p);
}

dsv4_status dsv4_sparse_mqa_decode(const dsv4_mqa_args *a, void *ws, size_t ws_bytes, dsv4_stream stream) {
  MqaLaunch p;
  const dsv4_status s = mqa_launch_args(a, &p);
  if (s != DSV4_OK) return s;
  const size_t need = mqa_workspace_bytes(p);
  if (need > 0 && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))) return DSV4_ERR_INVALID_ARG;
  return to_status(launch_mqa(p, ws, static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------------------------------
namespace {

struct HybridPlan {
  PrologueLaunch pro;
  IndexerLaunch ix;
  MqaLaunch mq;
  bool c4;
  size_t idx_bytes, ix_bytes, mq_bytes;  // workspace: selected entries, indexer, attention
};

dsv4_status hybrid_plan(const dsv4_layer *L, const dsv4_step *S, int32_t batch, HybridPlan *hp) {
  if (!L) return DSV4_ERR_INVALID_ARG;
  const bool c4 = L->kind == DSV4_LAYER_C4;
  if (!c4 && L->kind != DSV4_LAYER_C128) return DSV4_ERR_INVALID_ARG;
  if (batch <= 0 || batch > 65535 || L->heads <= 0 || L->dim <= 0) return DSV4_ERR_INVALID_ARG;
  if (!L->gamma || !valid_state(L->state) || !valid_cache(L->cache) || !valid_ring(L->ring))
    return DSV4_ERR_INVALID_ARG;
  if (L->state.m != L->cache.m || L->state.dim != L->dim || L->cache.dim != L->dim || L->ring.dim != L->dim)
    return DSV4_ERR_INVALID_ARG;
  if (L->cache.dtype != L->ring.dtype || L->cache.dtype == DSV4_FP4E2M1) return DSV4_ERR_UNSUPPORTED;
  if (!valid_rope(L->rope, L->dim) || !(L->eps >= 0.f)) return DSV4_ERR_INVALID_ARG;
  if (!valid_pool_dim(L->dim)) return DSV4_ERR_UNSUPPORTED;
  if (c4) {
    if (L->topk <= 0 || L->idx_heads <= 0 || L->idx_dim <= 0 || !L->gamma_idx) return DSV4_ERR_INVALID_ARG;
    if (!valid_state(L->idx_state) || !valid_cache(L->idx_cache)) return DSV4_ERR_INVALID_ARG;
    if (L->idx_state.m != L->state.m || L->idx_cache.m != L->state.m || L->idx_state.dim != L->idx_dim ||
        L->idx_cache.dim != L->idx_dim)
      return DSV4_ERR_INVALID_ARG;
    if (L->idx_rope_dims < 0 || L->idx_rope_dims % 2 || L->idx_rope_dims > L->idx_dim) return DSV4_ERR_INVALID_ARG;
    if (!valid_pool_dim(L->idx_dim)) return DSV4_ERR_UNSUPPORTED;
  }
  *hp = HybridPlan{};
  hp->c4 = c4;
  PrologueLaunch &pr = hp->pro;
  pr.B = batch;
  pr.gamma = L->gamma;
  pr.eps = L->eps;
  pr.rope_dims = L->rope.rope_dims;
  pr.rope_base = L->rope.rope_base;
  pr.state = L->state.buf;
  pr.m = L->state.m;
  pr.D = L->dim;
  pr.G = L->state.gate_dim;
  pr.pages = L->cache.pages;
  pr.scales = L->cache.scales;
  pr.block_table = L->cache.block_table;
  pr.num_pages = L->cache.num_pages;
  pr.max_blocks = L->cache.max_blocks;
  pr.cache_dt = L->cache.dtype;
  pr.ring_rows = L->ring.rows;
  pr.ring_scales = L->ring.scales;
  pr.W = L->ring.window;
  pr.ring_dt = L->ring.dtype;
  if (c4) {
    pr.gamma_idx = L->gamma_idx;
    pr.idx_rope_dims = L->idx_rope_dims;
    pr.idx_state = L->idx_state.buf;
    pr.idx_D = L->idx_dim;
    pr.idx_G = L->idx_state.gate_dim;
    pr.idx_pages = L->idx_cache.pages;
    pr.idx_scales = L->idx_cache.scales;
    pr.idx_block_table = L->idx_cache.block_table;
    pr.idx_num_pages = L->idx_cache.num_pages;
    pr.idx_max_blocks = L->idx_cache.max_blocks;
    pr.idx_dt = L->idx_cache.dtype;
  }
  IndexerLaunch &ix = hp->ix;
  if (c4) {
    ix.B = batch;
    ix.H = L->idx_heads;
    ix.Dq = L->idx_dim;
    ix.k = L->topk;
    ix.k_pages = L->idx_cache.pages;
    ix.k_scales = L->idx_cache.scales;
    ix.block_table = L->idx_cache.block_table;
    ix.num_pages = L->idx_cache.num_pages;
    ix.max_blocks = L->idx_cache.max_blocks;
    ix.m = L->idx_cache.m;
    ix.k_dt = L->idx_cache.dtype;
    ix.q_rope_dims = L->q_idx_rope ? L->idx_rope_dims : 0;
    ix.rope_base = L->rope.rope_base;
    if (ix.k > 2048 || static_cast<int64_t>(ix.H) * ix.Dq > 8192 || ix.k_dt == DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
  }
  MqaLaunch &mq = hp->mq;
  mq.B = batch;
  mq.H = L->heads;
  mq.D = L->dim;
  mq.pages = L->cache.pages;
  mq.scales = L->cache.scales;
  mq.block_table = L->cache.block_table;
  mq.num_pages = L->cache.num_pages;
  mq.max_blocks = L->cache.max_blocks;
  mq.m = L->cache.m;
  mq.kv_dt = L->cache.dtype;
  mq.k = c4 ? L->topk : 0;
  mq.ring_rows = L->ring.rows;
  mq.ring_scales = L->ring.scales;
  mq.W = L->ring.window;
  mq.softmax_scale = L->softmax_scale;
  mq.rope_dims = L->rope.rope_dims;
  mq.rope_base = L->rope.rope_base;
  mq.q_norm_gamma = L->gamma_q;
  mq.q_norm_eps = L->eps;
  if (mq.D > 1024 || mq.D % 32 != 0) return DSV4_ERR_UNSUPPORTED;
  if (S) {
    if (S->batch != batch || !S->pos || !S->kv || !S->gate || !S->q || !S->out) return DSV4_ERR_INVALID_ARG;
    if (S->kv_dtype != DSV4_F32 && S->kv_dtype != DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
    if (S->q_dtype != DSV4_F32 && S->q_dtype != DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
    if (!valid_dtype(S->out_dtype)) return DSV4_ERR_UNSUPPORTED;
    if (S->out_dtype == DSV4_FP8E4M3 && (!S->out_scales || L->dim % kOutBlock != 0)) return DSV4_ERR_INVALID_ARG;
    if (!aligned16(S->q) || !aligned16(S->out)) return DSV4_ERR_INVALID_ARG;
    pr.pos = S->pos;
    pr.kv_dt = S->kv_dtype;
    pr.kv = S->kv;
    pr.gate = S->gate;
    pr.d_status = S->d_status;
    if (c4) {
      if (!S->idx_kv || !S->idx_gate || !S->q_idx || !S->w) return DSV4_ERR_INVALID_ARG;
      if (S->q_idx_dtype != DSV4_F32 && S->q_idx_dtype != DSV4_FP8E4M3) return DSV4_ERR_UNSUPPORTED;
      if (S->w_dtype != DSV4_F32 && S->w_dtype != DSV4_BF16) return DSV4_ERR_UNSUPPORTED;
      if (L->q_idx_rope && L->idx_rope_dims > 0 && S->q_idx_dtype != DSV4_F32) return DSV4_ERR_UNSUPPORTED;
      if (!aligned16(S->q_idx)) return DSV4_ERR_INVALID_ARG;
      pr.idx_kv = S->idx_kv;
      pr.idx_gate = S->idx_gate;
      ix.q = S->q_idx;
      ix.q_dt = S->q_idx_dtype;
      ix.q_scale = S->q_idx_scale;
      ix.w = S->w;
      ix.w_dt = S->w_dtype;
      ix.pos = S->pos;
      ix.n_entries = nullptr;
      ix.scores = nullptr;
      ix.d_status = S->d_status;
    }
    mq.q = S->q;
    mq.q_dt = S->q_dtype;
    mq.pos = S->pos;
    mq.n_entries = nullptr;
    mq.out = S->out;
    mq.out_dt = S->out_dtype;
    mq.out_scales = S->out_scales;
    mq.lse = nullptr;
    mq.d_status = S->d_status;
  } else {
    // sizing only: the dtype-dependent choices follow the typical step
    ix.q_dt = DSV4_FP8E4M3;
    mq.q_dt = DSV4_BF16;
  }
  hp->idx_bytes = c4 ? align_up(static_cast<size_t>(batch) * L->topk * sizeof(int32_t), 256) : 0;
  hp->ix_bytes = c4 ? align_up(indexer_workspace_bytes(ix), 256) : 0;
  hp->mq_bytes = align_up(mqa_workspace_bytes(mq), 256);
  return DSV4_OK;
}

}  // namespace

size_t dsv4_hybrid_decode_workspace_size(const dsv4_layer *layer, int32_t batch) {
  HybridPlan hp;
  if (hybrid_plan(layer, nullptr, batch, &hp) != DSV4_OK) return 0;
  // the indexer's tensor-core and CUDA-core paths need different candidate space: take the larger
  size_t ix = hp.ix_bytes;
  if (hp.c4) {
    IndexerLaunch alt = hp.ix;
    alt.q_dt = DSV4_F32;
    ix = ix > align_up(indexer_workspace_bytes(alt), 256) ? ix : align_up(indexer_workspace_bytes(alt), 256);
  }
  MqaLaunch alt = hp.mq;
  alt.q_dt = DSV4_F32;
  size_t mq = hp.mq_bytes > align_up(mqa_workspace_bytes(alt), 256) ? hp.mq_bytes : align_up(mqa_workspace_bytes(alt), 256);
  return hp.idx_bytes + ix + mq;
}

dsv4_status dsv4_hybrid_decode(const dsv4_layer *layer, const dsv4_step *step, void *ws, size_t ws_bytes,
                               dsv4_stream stream) {
  if (!step) return DSV4_ERR_INVALID_ARG;
  HybridPlan hp;
  const dsv4_status s = hybrid_plan(layer, step, step->batch, &hp);
  if (s != DSV4_OK) return s;
  const size_t need = hp.idx_bytes + hp.ix_bytes + hp.mq_bytes;
  if (need > 0 && (!ws || ws_bytes < need || (reinterpret_cast<uintptr_t>(ws) & 255u))) return DSV4_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char *w = static_cast<char *>(ws);
  void *mq_ws = w + hp.idx_bytes + hp.ix_bytes;
  void *ix_ws = w + hp.idx_bytes;
  cudaError_t e = cudaSuccess;
  if (hp.c4) {
    int32_t *idx = step->topk_idx ? step->topk_idx : reinterpret_cast<int32_t *>(w);
    hp.ix.idx = idx;
    hp.ix.release_next = true;  // the attention follows in this call
    hp.mq.idx = idx;
  }
  if (hp.c4 && indexer_uses_tensor_cores(hp.ix)) {
    // indexer (the entries before this step's append) -> prologue and query preparation,
    // beside it -> top-k (which scores the appended entry) -> attention
    hp.ix.before_append = true;
    e = launch_indexer_part(hp.ix, ix_ws, st, 1);
    if (e != cudaSuccess) return to_status(e);
    e = launch_decode_prologue(hp.pro, st);
    if (e != cudaSuccess) return to_status(e);
    e = launch_mqa_query(hp.mq, mq_ws, st);
    if (e != cudaSuccess) return to_status(e);
    e = launch_indexer_part(hp.ix, ix_ws, st, 2);
    if (e != cudaSuccess) return to_status(e);
  } else {
    // prologue -> query preparation (beside it) -> (C4: indexer -> top-k) -> attention
    e = launch_decode_prologue(hp.pro, st);
    if (e != cudaSuccess) return to_status(e);
    e = launch_mqa_query(hp.mq, mq_ws, st);
    if (e != cudaSuccess) return to_status(e);
    if (hp.c4) {
      e = launch_indexer_topk(hp.ix, ix_ws, st);
      if (e != cudaSuccess) return to_status(e);
    }
  }
  e = launch_mqa_attention(hp.mq, mq_ws, st);
  return to_status(e);
}

}  // extern "C"

// ------------------------------------------------------------------------------------
// Indexer top-k on library-owned scratch. For callers that cannot allocate: a host
// program without a device allocator of its own, or a decode loop that must not stall on
// cudaMalloc/cudaFree. The scratch is a file-scope device array; its address is resolved
// once per device and handed to the same launcher dsv4_indexer_topk uses.
namespace {

static __device__ __align__(256) unsigned char noalloc_scratch[DSV4_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;

// Device address of noalloc_scratch on the current device. The first call on a device
// resolves it (cudaGetSymbolAddress may load the module, which must not happen inside a
// stream capture) and caches the SM count, so later calls do no set-up work at all.
dsv4_status noalloc_scratch_address(void **out) {
  static std::mutex mu;
  static void *addr[kMaxDevices] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return to_status(cudaErrorInvalidDevice);
  if (dev < 0 || dev >= kMaxDevices) return DSV4_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, noalloc_scratch);
    if (e != cudaSuccess) return to_status(e);
    if (!p || (reinterpret_cast<uintptr_t>(p) & 255u)) return DSV4_ERR_CUDA;
    sm_count();
    addr[dev] = p;
  }
  *out = addr[dev];
  return DSV4_OK;
}

}  // namespace

extern "C" dsv4_status dsv4_indexer_topk_noalloc(const dsv4_indexer_args *a, dsv4_stream stream) {
  IndexerLaunch p;
  const dsv4_status s = indexer_launch_args(a, &p);
  if (s != DSV4_OK) return s;
  if (indexer_workspace_bytes(p) > DSV4_NOALLOC_SCRATCH_BYTES) return DSV4_ERR_SCRATCH_LIMIT;
  void *ws = nullptr;
  const dsv4_status r = noalloc_scratch_address(&ws);
  if (r != DSV4_OK) return r;
  // the launcher zeroes the candidate counts at the head of ws on `stream` itself
  return to_status(launch_indexer_topk(p, ws, static_cast<cudaStream_t>(stream)));
}
