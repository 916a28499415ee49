// KV compressor, window-key insert and the per-step state updates of a decode step.
//
// Compressor (step (1) of the decode method; vLLM "fused compressor + RMSNorm + RoPE +
// cache insert", SGLang "Flash Compressor"): for a completed block b of m tokens,
//   e_c   = sum_t softmax_t(g_{t,c}) * kv_{t,c}            (per channel, over the block)
//   e     = e / sqrt(mean(e^2) + eps) * gamma
//   e     = RoPE at position b*m on the last rope_dims dims (adjacent pairs)
//   entry b of the paged cache = e rounded to the cache dtype (fp8: one scale per row).
// Window key (vLLM "Q-norm + KV RoPE + K insert", K part): RoPE_t(RMSNorm(kv_t)), slot t % W.
//
// The work is bandwidth-bound: each CTA (256 threads) streams one block's m x (D + G)
// inputs with 16-byte loads, pools in fp32 registers split over token slices, merges the
// slices in shared memory, and finishes (norm, rotation, rounding, store) in one pass.
#include "common.cuh"
#include "internal.h"

namespace dsv4 {

namespace {

constexpr int kThreads = 256;
constexpr int kMaxD = 2048;  // channels of one compressed vector

struct SeqRange {
  int64_t p0, p1;  // new positions [p0, p1)
  int64_t row0;    // input row of position p0
};

__device__ __forceinline__ SeqRange seq_range(const int32_t *cu, const int32_t *start, int s) {
  SeqRange r;
  r.row0 = cu[s];
  r.p0 = start[s];
  r.p1 = r.p0 + (cu[s + 1] - cu[s]);
  return r;
}

// Where token t of a block comes from: the float32 state ring (earlier calls) or the
// caller's input rows (this call).
struct TokenSource {
  const float *state;  // [m][D+G] of this sequence
  const void *kv;      // [*][D] input rows
  const void *gate;    // [*][G]
  dsv4_dtype kv_dt;
  int64_t p0, row0;    // positions >= p0 are input row row0 + (t - p0)
  int m, D, G;
};

// Softmax-gated pool of block b into e[0..D) (shared memory, float32).
// Threads are split into token slices x channel groups of 8; each thread keeps an online
// (max, sum, weighted sum) per channel, and the slices are merged in shared memory.
__device__ void pool_block(const TokenSource &src, int64_t b, float *e, float *scratch /*3*kMaxD*/) {
  const int D = src.D, G = src.G, m = src.m;
  const int groups = D / 8;
  const int slices = kThreads / groups;  // >= 1 since D <= kMaxD
  const int tid = threadIdx.x;
  const int slice = tid / groups, cg = tid % groups;
  float mx[8], l[8], acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) { mx[i] = -INFINITY; l[i] = 0.f; acc[i] = 0.f; }
  if (slice < slices) {
    for (int u = slice; u < m; u += slices) {
      const int64_t t = b * m + u;
      float v[8], g[8];
      if (t < src.p0) {
        const float *row = src.state + static_cast<size_t>(t % m) * (D + G);
        if (G == D) {  // rows of 2D floats: 16-byte aligned
          load_row_f<8>(row, DSV4_F32, static_cast<size_t>(cg) * 8, v);
          load_row_f<8>(row + D, DSV4_F32, static_cast<size_t>(cg) * 8, g);
        } else {  // rows of D + 1 floats: scalar loads
          const float g0 = row[D];
#pragma unroll
          for (int i = 0; i < 8; ++i) { v[i] = row[cg * 8 + i]; g[i] = g0; }
        }
      } else {
        const size_t r = static_cast<size_t>(src.row0 + (t - src.p0));
        load_row_f<8>(src.kv, src.kv_dt, r * D + cg * 8, v);
        if (G == D) {
          load_row_f<8>(src.gate, src.kv_dt, r * G + cg * 8, g);
        } else {
          const float g0 = load_one_f(src.gate, src.kv_dt, r * G);
#pragma unroll
          for (int i = 0; i < 8; ++i) g[i] = g0;
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        if (g[i] > mx[i]) {
          const float a = expf(mx[i] - g[i]);
          acc[i] = acc[i] * a + v[i];
          l[i] = l[i] * a + 1.f;
          mx[i] = g[i];
        } else {
          const float w = expf(g[i] - mx[i]);
          acc[i] += w * v[i];
          l[i] += w;
        }
      }
    }
  }
  float *smx = scratch, *sl = scratch + kMaxD, *sacc = scratch + 2 * kMaxD;
  __syncthreads();
  if (slice < slices) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int idx = slice * D + cg * 8 + i;  // slices * D <= kThreads * 8 = kMaxD
      smx[idx] = mx[i];
      sl[idx] = l[i];
      sacc[idx] = acc[i];
    }
  }
  __syncthreads();
  for (int c = tid; c < D; c += kThreads) {
    float M = -INFINITY;
    for (int s = 0; s < slices; ++s) M = fmaxf(M, smx[s * D + c]);
    float L = 0.f, A = 0.f;
    for (int s = 0; s < slices; ++s) {
      const float ms = smx[s * D + c];
      if (ms == -INFINITY) continue;
      const float w = expf(ms - M);
      L += w * sl[s * D + c];
      A += w * sacc[s * D + c];
    }
    e[c] = A / L;
  }
  __syncthreads();
}

// RMSNorm(e) * gamma, RoPE at `rope_pos`, round into `dt`, store to `row` (+ *scale_out).
// e: shared float[D]; red: shared float[32]. Every thread of the CTA calls this.
__device__ void finish_and_store(float *e, int D, const float *gamma, float eps, int64_t rope_pos, int rope_dims,
                                 double rope_theta1, dsv4_dtype dt, void *row, float *scale_out, float *red) {
  const int tid = threadIdx.x;
  float ss = 0.f;
  for (int c = tid; c < D; c += kThreads) ss += e[c] * e[c];
  ss = block_sum(ss, red);
  const float rs = 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
  __syncthreads();
  for (int c = tid; c < D; c += kThreads) e[c] = e[c] * rs * gamma[c];
  __syncthreads();
  const int half = rope_dims / 2;
  for (int i = tid; i < half; i += kThreads) {
    float cs, sn;
    rope_cos_sin(rope_pos, i, rope_theta1, &cs, &sn);
    const int c0 = D - rope_dims + 2 * i;
    const float x0 = e[c0], x1 = e[c0 + 1];
    e[c0] = x0 * cs - x1 * sn;
    e[c0 + 1] = x0 * sn + x1 * cs;
  }
  __syncthreads();
  if (dt == DSV4_F32) {
    float *o = static_cast<float *>(row);
    for (int c = tid; c < D; c += kThreads) o[c] = e[c];
  } else if (dt == DSV4_BF16) {
    uint16_t *o = static_cast<uint16_t *>(row);
    for (int c = tid; c < D; c += kThreads) o[c] = float_to_bf16_bits(e[c]);
  } else {
    float am = 0.f;
    for (int c = tid; c < D; c += kThreads) am = fmaxf(am, fabsf(e[c]));
    am = block_max(am, red);
    const float scale = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
    const float inv = am > 0.f ? __fdiv_rn(448.0f, am) : 1.0f;
    uint8_t *o = static_cast<uint8_t *>(row);
    for (int c2 = tid; c2 < D / 2; c2 += kThreads) {
      const uint16_t pr = float2_to_e4m3x2(__fmul_rn(e[2 * c2], inv), __fmul_rn(e[2 * c2 + 1], inv));
      *reinterpret_cast<uint16_t *>(o + 2 * c2) = pr;
    }
    if (tid == 0 && scale_out) *scale_out = scale;
  }
  __syncthreads();
}

// Paged-cache row of entry j of sequence s, or nullptr (reported) if out of range.
__device__ __forceinline__ void *cache_row(void *pages, float *scales, const int32_t *bt, int num_pages,
                                           int max_blocks, int m, int D, dsv4_dtype dt, int s, int64_t j,
                                           float **scale_ptr, uint32_t *d_status) {
  const int per_page = DSV4_PAGE_POSITIONS / m;
  const int64_t lb = j / per_page;
  if (j < 0 || lb >= max_blocks) {
    report(d_status, DSV4_DEV_BAD_LENGTH);
    return nullptr;
  }
  const int page = bt[static_cast<size_t>(s) * max_blocks + lb];
  if (page < 0 || page >= num_pages) {
    report(d_status, DSV4_DEV_BAD_PAGE);
    return nullptr;
  }
  const size_t r = static_cast<size_t>(page) * per_page + static_cast<size_t>(j % per_page);
  *scale_ptr = scales ? scales + r : nullptr;
  return static_cast<char *>(pages) + r * D * dtype_size(dt);
}

// items of sequence s: one per completed block, at least one (the state-tail write)
__device__ __forceinline__ int64_t compress_items(const SeqRange &r, int m) {
  const int64_t c = r.p1 / m - r.p0 / m;
  return c > 1 ? c : 1;
}

__global__ void __launch_bounds__(kThreads) compress_kernel(const CompressLaunch p) {
  pdl_wait();  // the only kernel of its call: it releases nothing early
  extern __shared__ __align__(16) float smem[];
  float *scratch = smem;             // 3 * kMaxD
  float *e = smem + 3 * kMaxD;       // kMaxD
  float *red = e + kMaxD;            // 32
  long long *prefix = reinterpret_cast<long long *>(red + 32);  // B + 1
  const int tid = threadIdx.x;
  if (tid == 0) {
    long long acc = 0;
    for (int s = 0; s < p.B; ++s) {
      prefix[s] = acc;
      acc += compress_items(seq_range(p.cu_seqlens, p.start_pos, s), p.m);
    }
    prefix[p.B] = acc;
  }
  __syncthreads();
  const long long total = prefix[p.B];
  for (long long item = blockIdx.x; item < total; item += gridDim.x) {
    int lo = 0, hi = p.B - 1;  // last s with prefix[s] <= item
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int s = lo;
    const int64_t i = item - prefix[s];
    const SeqRange r = seq_range(p.cu_seqlens, p.start_pos, s);
    float *st = p.state + static_cast<size_t>(s) * p.m * (p.D + p.G);
    const bool has_block = (r.p1 / p.m - r.p0 / p.m) > i;
    if (has_block) {
      const int64_t b = r.p0 / p.m + i;
      TokenSource src{st, p.kv, p.gate, p.kv_dt, r.p0, r.row0, p.m, p.D, p.G};
      pool_block(src, b, e, scratch);
      float *sp = nullptr;
      void *row = cache_row(p.pages, p.scales, p.block_table, p.num_pages, p.max_blocks, p.m, p.D, p.cache_dt, s, b,
                            &sp, p.d_status);
      if (row != nullptr)  // uniform over the CTA
        finish_and_store(e, p.D, p.gamma, p.eps, b * p.m, p.rope_dims, p.rope_theta1, p.cache_dt, row, sp, red);
    }
    if (i == 0) {
      // the state ring keeps the latest m tokens (slot t % m); written after the first
      // block, the only one that may read ring slots, has been pooled
      __syncthreads();
      int64_t t0 = r.p1 - p.m;
      if (t0 < r.p0) t0 = r.p0;
      const int width = p.D + p.G;
      for (int64_t t = t0; t < r.p1; ++t) {
        const size_t rin = static_cast<size_t>(r.row0 + (t - r.p0));
        float *dst = st + static_cast<size_t>(t % p.m) * width;
        for (int c = tid; c < p.D; c += kThreads) dst[c] = load_one_f(p.kv, p.kv_dt, rin * p.D + c);
        for (int c = tid; c < p.G; c += kThreads) dst[p.D + c] = load_one_f(p.gate, p.kv_dt, rin * p.G + c);
      }
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(kThreads) swa_insert_kernel(const SwaLaunch p) {
  pdl_wait();  // the only kernel of its call: it releases nothing early
  __shared__ float e[kMaxD];
  __shared__ float red[32];
  const int s = blockIdx.y;
  const SeqRange r = seq_range(p.cu_seqlens, p.start_pos, s);
  int64_t t0 = r.p1 - p.W;
  if (t0 < r.p0) t0 = r.p0;
  const int64_t t = t0 + blockIdx.x;
  if (t >= r.p1) return;
  const size_t rin = static_cast<size_t>(r.row0 + (t - r.p0));
  for (int c = threadIdx.x; c < p.D; c += kThreads) e[c] = load_one_f(p.kv, p.kv_dt, rin * p.D + c);
  __syncthreads();
  const size_t slot = static_cast<size_t>(s) * p.W + static_cast<size_t>(t % p.W);
  void *row = static_cast<char *>(p.rows) + slot * p.D * dtype_size(p.ring_dt);
  finish_and_store(e, p.D, p.gamma, p.eps, t, p.rope_dims, p.rope_theta1, p.ring_dt, row,
                   p.scales ? p.scales + slot : nullptr, red);
}

// One decode step's updates. blockIdx.y: 0 = window insert, 1 = main compressor append,
// 2 = indexer-key compressor append.
__global__ void __launch_bounds__(kThreads) decode_prologue_kernel(const PrologueLaunch p) {
  pdl_wait();
  pdl_launch_dependents();
  extern __shared__ __align__(16) float smem[];
  float *scratch = smem;
  float *e = smem + 3 * kMaxD;
  float *red = e + kMaxD;
  const int s = blockIdx.x, role = blockIdx.y;
  const int tid = threadIdx.x;
  const int64_t pos = p.pos[s];
  if (pos < 0) {
    if (tid == 0) report(p.d_status, DSV4_DEV_BAD_LENGTH);
    return;
  }
  if (role == 0) {
    for (int c = tid; c < p.D; c += kThreads) e[c] = load_one_f(p.kv, p.kv_dt, static_cast<size_t>(s) * p.D + c);
    __syncthreads();
    const size_t slot = static_cast<size_t>(s) * p.W + static_cast<size_t>(pos % p.W);
    void *row = static_cast<char *>(p.ring_rows) + slot * p.D * dtype_size(p.ring_dt);
    finish_and_store(e, p.D, p.gamma, p.eps, pos, p.rope_dims, p.rope_theta1, p.ring_dt, row,
                     p.ring_scales ? p.ring_scales + slot : nullptr, red);
    return;
  }
  const bool idx = role == 2;
  const int D = idx ? p.idx_D : p.D, G = idx ? p.idx_G : p.G, m = p.m;
  float *st = (idx ? p.idx_state : p.state) + static_cast<size_t>(s) * m * (D + G);
  const void *kv = idx ? p.idx_kv : p.kv;
  const void *gate = idx ? p.idx_gate : p.gate;
  float *dst = st + static_cast<size_t>(pos % m) * (D + G);
  for (int c = tid; c < D; c += kThreads) dst[c] = load_one_f(kv, p.kv_dt, static_cast<size_t>(s) * D + c);
  for (int c = tid; c < G; c += kThreads) dst[D + c] = load_one_f(gate, p.kv_dt, static_cast<size_t>(s) * G + c);
  if ((pos + 1) % m != 0) return;
  __syncthreads();
  const int64_t b = (pos + 1) / m - 1;
  TokenSource src{st, nullptr, nullptr, p.kv_dt, b * m + m, 0, m, D, G};  // whole block from the ring
  pool_block(src, b, e, scratch);
  float *sp = nullptr;
  void *row = idx ? cache_row(p.idx_pages, p.idx_scales, p.idx_block_table, p.idx_num_pages, p.idx_max_blocks, m, D,
                              p.idx_dt, s, b, &sp, p.d_status)
                  : cache_row(p.pages, p.scales, p.block_table, p.num_pages, p.max_blocks, m, D, p.cache_dt, s, b, &sp,
                              p.d_status);
  if (row != nullptr)
    finish_and_store(e, D, idx ? p.gamma_idx : p.gamma, p.eps, b * m, idx ? p.idx_rope_dims : p.rope_dims,
                     idx ? p.idx_rope_theta1 : p.rope_theta1, idx ? p.idx_dt : p.cache_dt, row, sp, red);
}

constexpr size_t kPoolSmem = (4 * kMaxD + 32) * sizeof(float);

}  // namespace

cudaError_t launch_compress(const CompressLaunch &p0, cudaStream_t st) {
  CompressLaunch p = p0;
  p.rope_theta1 = rope_theta1(p.rope_base, p.rope_dims);
  const size_t smem = kPoolSmem + (p.B + 1) * sizeof(long long);
  cudaError_t e = cudaFuncSetAttribute(compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const long long upper = static_cast<long long>(p.total_tokens) / p.m + p.B;
  const long long cap = static_cast<long long>(sm_count()) * 8;
  const int grid = static_cast<int>(upper < cap ? (upper > 0 ? upper : 1) : cap);
  return launch_pdl(compress_kernel, dim3(grid), dim3(kThreads), smem, st, 1, p);
}

cudaError_t launch_swa_insert(const SwaLaunch &p0, cudaStream_t st) {
  SwaLaunch p = p0;
  p.rope_theta1 = rope_theta1(p.rope_base, p.rope_dims);
  dim3 grid(p.W, p.B);
  return launch_pdl(swa_insert_kernel, grid, dim3(kThreads), 0, st, 1, p);
}

cudaError_t launch_decode_prologue(const PrologueLaunch &p0, cudaStream_t st) {
  PrologueLaunch p = p0;
  p.rope_theta1 = rope_theta1(p.rope_base, p.rope_dims);
  p.idx_rope_theta1 = rope_theta1(p.rope_base, p.idx_rope_dims);
  cudaError_t e =
      cudaFuncSetAttribute(decode_prologue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPoolSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.B, p.idx_D > 0 ? 3 : 2);
  return launch_pdl(decode_prologue_kernel, grid, dim3(kThreads), kPoolSmem, st, 1, p);
}

}  // namespace dsv4
