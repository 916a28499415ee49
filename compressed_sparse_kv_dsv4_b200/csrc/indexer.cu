// Lightning indexer + top-k (step (2) of the decode method; "DeepSeek Sparse Attention
// over compressed tokens" in the vLLM post, "Lightning TopK" in the SGLang blog).
//
//   s_j = sum_h w_h * ReLU(q_h . k_j)       for every visible C4 entry j
//   keep the k largest s_j (ties to the lower j)
//
// Tensor-core path (fp8 keys, 128-dim, the C4 layers): a persistent kernel, one CTA per
// SM, over the flattened (sequence, 128-entry tile) space. Warp 0 streams key tiles with
// TMA (two 8 KB page boxes per tile, 128B swizzle) into an 8-stage ring; warp 1 issues
// tcgen05.mma kind::f8f6f4 (M = 128 entries, N = H heads, K = 128) into a double-buffered
// TMEM accumulator; warps 2-5 read the accumulator back (tcgen05.ld), apply ReLU, the
// per-head weights w_h * scale_q[h] and the per-entry key scale, and keep a running
// top-k in shared memory (threshold filter + radix-select compaction). Each CTA writes at
// most k candidates per sequence segment; a small select kernel merges them.
//
// The scale handling relies on ReLU(a * x) = a * ReLU(x) for a > 0:
//   s_j = scale_k[j] * sum_h (w_h * scale_q[h]) * ReLU(q8_h . k8_j).
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace dsv4 {

namespace {

constexpr int kTile = 128;      // entries per tile = MMA M
constexpr int kRowBytes = 128;  // fp8 key row = 128 dims
constexpr int kStages = 8;
constexpr int kCap = 2048;      // candidate buffer of one CTA segment
constexpr int kMaxK = 1024;     // largest k of the tensor-core path
constexpr int kTcThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kSelThreads = 1024;
constexpr int kMaxSortK = 2048;

__device__ __forceinline__ int64_t visible_entries(const int32_t *n_entries, const int32_t *pos, int m, int b,
                                                   int64_t capacity, uint32_t *d_status, bool report_it) {
  int64_t n = n_entries ? static_cast<int64_t>(n_entries[b]) : (static_cast<int64_t>(pos[b]) + 1) / m;
  if (n < 0) n = 0;
  if (n > capacity) {
    if (report_it) report(d_status, DSV4_DEV_BAD_LENGTH);
    n = capacity;
  }
  return n;
}

// ------------------------------------------------------------------------------------
// CUDA-core scoring: one thread per entry; writes every entry's key to the candidate list.

__global__ void __launch_bounds__(256) indexer_simt_kernel(const IndexerLaunch p, unsigned long long *cand,
                                                           int64_t stride, int *cand_count) {
  extern __shared__ float sq[];  // [H][Dq] query, then [H] coefficients
  const int b = blockIdx.y;
  const int per_page = DSV4_PAGE_POSITIONS / p.m;
  const int64_t capacity = static_cast<int64_t>(p.max_blocks) * per_page;
  const int64_t n = visible_entries(p.n_entries, p.pos, p.m, b, capacity, p.d_status, blockIdx.x == 0 && threadIdx.x == 0);
  if (blockIdx.x == 0 && threadIdx.x == 0) cand_count[b] = static_cast<int>(n);
  if (static_cast<int64_t>(blockIdx.x) * blockDim.x >= n) return;
  const int H = p.H, Dq = p.Dq;
  float *coef = sq + H * Dq;
  for (int i = threadIdx.x; i < H * Dq; i += blockDim.x) {
    const size_t off = static_cast<size_t>(b) * H * Dq + i;
    float v = load_one_f(p.q, p.q_dt, off);
    if (p.q_dt == DSV4_FP8E4M3 && p.q_scale) v *= p.q_scale[static_cast<size_t>(b) * H + i / Dq];
    sq[i] = v;
  }
  for (int h = threadIdx.x; h < H; h += blockDim.x) coef[h] = load_one_f(p.w, p.w_dt, static_cast<size_t>(b) * H + h);
  __syncthreads();
  if (p.q_rope_dims > 0) {
    const int half = p.q_rope_dims / 2;
    for (int t = threadIdx.x; t < H * half; t += blockDim.x) {
      const int h = t / half, i = t % half;
      float c, s;
      rope_cos_sin(p.pos[b], i, p.q_rope_dims, p.rope_base, &c, &s);
      float *x = sq + h * Dq + Dq - p.q_rope_dims + 2 * i;
      const float x0 = x[0], x1 = x[1];
      x[0] = x0 * c - x1 * s;
      x[1] = x0 * s + x1 * c;
    }
    __syncthreads();
  }
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t lb = j / per_page;
  const int page = p.block_table[static_cast<size_t>(b) * p.max_blocks + lb];
  unsigned long long key = 0;
  if (page < 0 || page >= p.num_pages) {
    report(p.d_status, DSV4_DEV_BAD_PAGE);
  } else {
    const size_t row = static_cast<size_t>(page) * per_page + static_cast<size_t>(j % per_page);
    const float ks = p.k_dt == DSV4_FP8E4M3 ? p.k_scales[row] : 1.0f;
    float s = 0.f;
    for (int h = 0; h < H; ++h) {
      float dot = 0.f;
      for (int c = 0; c < Dq; ++c) dot = fmaf(sq[h * Dq + c], load_one_f(p.k_pages, p.k_dt, row * Dq + c), dot);
      s = fmaf(coef[h], fmaxf(dot * ks, 0.f), s);
    }
    key = topk_key(s, static_cast<uint32_t>(j));
  }
  cand[static_cast<size_t>(b) * stride + j] = key;
}

// ------------------------------------------------------------------------------------
// Tensor-core scoring with a fused per-CTA top-k.

struct TcParams {
  CUtensorMap tmap_k;  // keys as [num_pages * per_page rows][128 bytes]
  CUtensorMap tmap_q;  // queries as [B * H rows][128 bytes]
  const float *k_scales;
  const int32_t *block_table;
  int num_pages, max_blocks, per_page, box_rows;
  const float *q_scale;
  const void *w;
  dsv4_dtype w_dt;
  int B, k, m;
  const int32_t *n_entries;
  const int32_t *pos;
  unsigned long long *cand;
  int64_t stride;
  int *cand_count;
  uint32_t *d_status;
};

template <int H>
struct alignas(1024) TcSmem {
  uint8_t stage[kStages][kTile * kRowBytes];
  uint8_t q[2][H * kRowBytes];
  unsigned long long cand[kCap];
  unsigned long long cand2[kMaxK];
  float coef[2][H];
  int hist[256];
  uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], qfull[2], qempty[2];
  unsigned long long thr, sel_prefix, sel_mask;
  uint32_t tmem_base;
  int abort_flag, stop, cnt, cnt2, out_base, sel_digit, sel_above, sel_count;
};

// Find the k largest of cand[0..cnt) (distinct 64-bit keys) by an MSB-first radix
// select over bytes; leaves (prefix, mask) so that kept = {key : (key & mask) >= prefix}
// has exactly k elements. Called by the 128 epilogue threads together.
template <int H>
__device__ void radix_select_smem(TcSmem<H> &S, int cnt, int k, int ep_tid) {
  unsigned long long prefix = 0, mask = 0;
  int need = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = ep_tid; i < 256; i += kEpiThreads) S.hist[i] = 0;
    named_bar_sync(1, kEpiThreads);
    for (int i = ep_tid; i < cnt; i += kEpiThreads) {
      const unsigned long long key = S.cand[i];
      if ((key & mask) == prefix) atomicAdd(&S.hist[(key >> shift) & 0xFF], 1);
    }
    named_bar_sync(1, kEpiThreads);
    if (ep_tid < 32) {
      const int lane = ep_tid;
      int c[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) { c[u] = S.hist[255 - lane * 8 - u]; tot += c[u]; }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += v;
      }
      int run = incl - tot;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (run < need && run + c[u] >= need) {
          S.sel_digit = 255 - lane * 8 - u;
          S.sel_above = run;
          S.sel_count = c[u];
        }
        run += c[u];
      }
    }
    named_bar_sync(1, kEpiThreads);
    const int digit = S.sel_digit, above = S.sel_above, cntd = S.sel_count;
    prefix |= static_cast<unsigned long long>(digit) << shift;
    mask |= 0xFFull << shift;
    need -= above;
    named_bar_sync(1, kEpiThreads);
    if (cntd == need) break;
  }
  if (ep_tid == 0) { S.sel_prefix = prefix; S.sel_mask = mask; }
  named_bar_sync(1, kEpiThreads);
}

// keep exactly the k best candidates; raise the insertion threshold
template <int H>
__device__ void compact(TcSmem<H> &S, int k, int ep_tid) {
  const int cnt = S.cnt;
  radix_select_smem(S, cnt, k, ep_tid);
  const unsigned long long prefix = S.sel_prefix, mask = S.sel_mask;
  if (ep_tid == 0) S.cnt2 = 0;
  named_bar_sync(1, kEpiThreads);
  for (int i = ep_tid; i < cnt; i += kEpiThreads) {
    const unsigned long long key = S.cand[i];
    if ((key & mask) >= prefix) {
      const int at = atomicAdd(&S.cnt2, 1);
      if (at < kMaxK) S.cand2[at] = key;
    }
  }
  named_bar_sync(1, kEpiThreads);
  const int kept = S.cnt2 < k ? S.cnt2 : k;
  for (int i = ep_tid; i < kept; i += kEpiThreads) S.cand[i] = S.cand2[i];
  named_bar_sync(1, kEpiThreads);
  if (ep_tid == 0) {
    S.cnt = kept;
    if (prefix > S.thr) S.thr = prefix;
  }
  named_bar_sync(1, kEpiThreads);
}

__device__ __forceinline__ int find_seq(const long long *prefix, int B, long long g) {
  int lo = 0, hi = B - 1;  // last b with prefix[b] <= g
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

template <int H>
__global__ void __launch_bounds__(kTcThreads, 1) indexer_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem<H> &S = *reinterpret_cast<TcSmem<H> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  long long *prefix = reinterpret_cast<long long *>(&S + 1);  // [B + 1] tiles before sequence b
  int64_t *nvis = reinterpret_cast<int64_t *>(prefix + p.B + 1);  // [B] visible entries
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t capacity = static_cast<int64_t>(p.max_blocks) * p.per_page;

  // ---- setup: barriers, TMEM, tile prefix over sequences
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.tfull[i], 1);
      mbar_init(&S.tempty[i], kEpiThreads / 32);
      mbar_init(&S.qfull[i], 1);
      mbar_init(&S.qempty[i], 1);
    }
    S.abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tmap_k);
    prefetch_tensormap(&p.tmap_q);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 2 * H);
    tmem_relinquish();
  }
  for (int b = tid; b < p.B; b += kTcThreads)
    nvis[b] = visible_entries(p.n_entries, p.pos, p.m, b, capacity, p.d_status, blockIdx.x == 0);
  __syncthreads();
  if (tid == 0) {
    long long acc = 0;
    for (int b = 0; b < p.B; ++b) {
      prefix[b] = acc;
      acc += (nvis[b] + kTile - 1) / kTile;
    }
    prefix[p.B] = acc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const long long T = prefix[p.B];
  const long long G = gridDim.x;
  const long long t0 = (T * blockIdx.x) / G, t1 = (T * (blockIdx.x + 1)) / G;

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int cur_b = -1, seg = -1;
      long long issued = 0;
      for (long long g = t0; g < t1; ++g) {
        const int b = find_seq(prefix, p.B, g);
        const long long lt = g - prefix[b];
        if (b != cur_b) {
          cur_b = b;
          ++seg;
          const int slot = seg & 1;
          if (seg >= 2 && !mbar_wait(&S.qempty[slot], ((seg >> 1) - 1) & 1, &S.abort_flag)) break;
          mbar_arrive_expect_tx(&S.qfull[slot], H * kRowBytes);
          tma_load_2d(S.q[slot], &p.tmap_q, &S.qfull[slot], 0, b * H);
        }
        const long long n = g - t0;
        const int s = static_cast<int>(n % kStages);
        const long long r = n / kStages;
        if (r >= 1 && !mbar_wait(&S.empty[s], static_cast<uint32_t>((r - 1) & 1), &S.abort_flag)) break;
        const int64_t e0 = lt * kTile;
        const int nbox = kTile / p.box_rows;
        int pages[kTile / 16];
        uint32_t bytes = 0;
        for (int h = 0; h < nbox; ++h) {
          const int64_t first = e0 + static_cast<int64_t>(h) * p.box_rows;
          pages[h] = -1;
          if (first < nvis[b]) {
            const int pg = p.block_table[static_cast<size_t>(b) * p.max_blocks + first / p.per_page];
            if (pg >= 0 && pg < p.num_pages) {
              pages[h] = pg * p.per_page + static_cast<int>(first % p.per_page);
              bytes += p.box_rows * kRowBytes;
            } else {
              report(p.d_status, DSV4_DEV_BAD_PAGE);
            }
          }
        }
        mbar_arrive_expect_tx(&S.full[s], bytes);
        for (int h = 0; h < nbox; ++h)
          if (pages[h] >= 0) tma_load_2d(S.stage[s] + h * p.box_rows * kRowBytes, &p.tmap_k, &S.full[s], 0, pages[h]);
        ++issued;
      }
      if (S.abort_flag) {
        // let loads already in flight land before the CTA leaves
        const long long from = issued > kStages ? issued - kStages : 0;
        for (long long n = from; n < issued; ++n) {
          volatile int dummy = 0;
          mbar_wait(&S.full[n % kStages], static_cast<uint32_t>((n / kStages) & 1), &dummy);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3(kTile, H);
      int cur_b = -1, seg = -1;
      for (long long g = t0; g < t1; ++g) {
        const int b = find_seq(prefix, p.B, g);
        if (b != cur_b) {
          cur_b = b;
          ++seg;
          if (!mbar_wait(&S.qfull[seg & 1], (seg >> 1) & 1, &S.abort_flag)) break;
        }
        const long long n = g - t0;
        const int s = static_cast<int>(n % kStages);
        if (!mbar_wait(&S.full[s], static_cast<uint32_t>((n / kStages) & 1), &S.abort_flag)) break;
        const int acc = static_cast<int>(n & 1);
        const long long ar = n >> 1;
        if (ar >= 1 && !mbar_wait(&S.tempty[acc], static_cast<uint32_t>((ar - 1) & 1), &S.abort_flag)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(S.stage[s]), b0 = smem_u32(S.q[seg & 1]);
#pragma unroll
        for (int kk = 0; kk < kRowBytes / 32; ++kk)
          mma_e4m3(tmem + acc * H, sw128_desc(a0 + kk * 32, 16, 1024), sw128_desc(b0 + kk * 32, 16, 1024), idesc,
                   kk > 0 ? 1u : 0u);
        mma_commit(&S.empty[s]);
        mma_commit(&S.tfull[acc]);
        const bool seg_end = (g + 1 == t1) || (find_seq(prefix, p.B, g + 1) != b);
        if (seg_end) mma_commit(&S.qempty[seg & 1]);
      }
    }
  } else {
    // ---------------- epilogue: scores + running top-k (warps 2..5)
    const int ep_tid = tid - 64;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    int cur_b = -1, seg = -1;
    for (long long g = t0; g < t1; ++g) {
      const int b = find_seq(prefix, p.B, g);
      const long long lt = g - prefix[b];
      if (b != cur_b) {
        cur_b = b;
        ++seg;
        for (int h = ep_tid; h < H; h += kEpiThreads) {
          const float qs = p.q_scale ? p.q_scale[static_cast<size_t>(b) * H + h] : 1.0f;
          S.coef[seg & 1][h] = load_one_f(p.w, p.w_dt, static_cast<size_t>(b) * H + h) * qs;
        }
        if (ep_tid == 0) { S.cnt = 0; S.thr = 1; }
        named_bar_sync(1, kEpiThreads);
      }
      const int64_t j = lt * kTile + row;
      float ks = 0.f;
      bool valid = j < nvis[b];
      if (valid) {
        const int pg = p.block_table[static_cast<size_t>(b) * p.max_blocks + j / p.per_page];
        valid = pg >= 0 && pg < p.num_pages;
        if (valid) ks = p.k_scales[static_cast<size_t>(pg) * p.per_page + static_cast<size_t>(j % p.per_page)];
      }
      const long long n = g - t0;
      const int acc = static_cast<int>(n & 1);
      bool ok = mbar_wait(&S.tfull[acc], static_cast<uint32_t>((n >> 1) & 1), &S.abort_flag);
      ok = __all_sync(0xFFFFFFFFu, ok);
      float score = 0.f;
      if (ok) {
        tc_fence_after();
        const float *cf = S.coef[seg & 1];
#pragma unroll
        for (int c0 = 0; c0 < H; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + acc * H + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) score = fmaf(cf[c0 + i], fmaxf(__uint_as_float(r[i]), 0.f), score);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&S.tempty[acc]);
      } else if (lane == 0) {
        S.abort_flag = 1;
      }
      score *= ks;
      const unsigned long long key = (ok && valid) ? topk_key(score, static_cast<uint32_t>(j)) : 0ull;
      named_bar_sync(1, kEpiThreads);
      if (ep_tid == 0) S.stop = S.abort_flag;
      named_bar_sync(1, kEpiThreads);
      if (S.stop) break;
      if (S.cnt > kCap - kEpiThreads) compact(S, p.k, ep_tid);
      const bool pass = key != 0ull && key >= S.thr;
      const unsigned bal = __ballot_sync(0xFFFFFFFFu, pass);
      int base = 0;
      if (lane == 0 && bal) base = atomicAdd(&S.cnt, __popc(bal));
      base = __shfl_sync(0xFFFFFFFFu, base, 0);
      if (pass) S.cand[base + __popc(bal & ((1u << lane) - 1u))] = key;
      const bool seg_end = (g + 1 == t1) || (find_seq(prefix, p.B, g + 1) != b);
      if (seg_end) {
        named_bar_sync(1, kEpiThreads);
        if (S.cnt > p.k) compact(S, p.k, ep_tid);
        const int nout = S.cnt;
        if (ep_tid == 0) S.out_base = atomicAdd(&p.cand_count[b], nout);
        named_bar_sync(1, kEpiThreads);
        const int base_out = S.out_base;
        if (base_out + nout > p.stride) {
          if (ep_tid == 0) report(p.d_status, DSV4_DEV_BAD_LENGTH);
        } else {
          for (int i = ep_tid; i < nout; i += kEpiThreads)
            p.cand[static_cast<size_t>(b) * p.stride + base_out + i] = S.cand[i];
        }
        named_bar_sync(1, kEpiThreads);
      }
    }
  }

  if (tid == 0 && S.abort_flag) report(p.d_status, DSV4_DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * H);
  }
}

// ------------------------------------------------------------------------------------
// Per-sequence select: the k best keys of the candidate list, sorted (score desc,
// index asc), written as entry indices (+ scores); -1 / -inf padding.

__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(const unsigned long long *cand, int64_t stride,
                                                                  const int *cand_count, int k, int32_t *idx,
                                                                  float *scores, uint32_t *d_status) {
  __shared__ int hist[256];
  __shared__ unsigned long long sorted[kMaxSortK];
  __shared__ int sel_digit, sel_above, sel_count, kept;
  const int b = blockIdx.x, tid = threadIdx.x;
  const unsigned long long *c = cand + static_cast<size_t>(b) * stride;
  int cnt = cand_count[b];
  if (cnt > stride) {
    if (tid == 0) report(d_status, DSV4_DEV_BAD_LENGTH);
    cnt = static_cast<int>(stride);
  }
  unsigned long long prefix = 0, mask = 0;
  if (cnt > k) {
    int need = k;
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int i = tid; i < cnt; i += kSelThreads) {
        const unsigned long long key = c[i];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFF], 1);
      }
      __syncthreads();
      if (tid < 32) {
        int cc[8], tot = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) { cc[u] = hist[255 - tid * 8 - u]; tot += cc[u]; }
        int incl = tot;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
          if (tid >= o) incl += v;
        }
        int run = incl - tot;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          if (run < need && run + cc[u] >= need) { sel_digit = 255 - tid * 8 - u; sel_above = run; sel_count = cc[u]; }
          run += cc[u];
        }
      }
      __syncthreads();
      prefix |= static_cast<unsigned long long>(sel_digit) << shift;
      mask |= 0xFFull << shift;
      need -= sel_above;
      const int cntd = sel_count;
      __syncthreads();
      if (cntd == need) break;
    }
  }
  int kp2 = 1;
  while (kp2 < k) kp2 <<= 1;
  if (tid == 0) kept = 0;
  for (int i = tid; i < kp2; i += kSelThreads) sorted[i] = 0ull;
  __syncthreads();
  for (int i = tid; i < cnt; i += kSelThreads) {
    const unsigned long long key = c[i];
    if (key != 0ull && (key & mask) >= prefix) {
      const int at = atomicAdd(&kept, 1);
      if (at < k) sorted[at] = key;
    }
  }
  __syncthreads();
  // bitonic sort, descending
  for (int size = 2; size <= kp2; size <<= 1) {
    for (int stride2 = size >> 1; stride2 > 0; stride2 >>= 1) {
      for (int i = tid; i < kp2; i += kSelThreads) {
        const int jx = i ^ stride2;
        if (jx > i) {
          const bool desc = (i & size) == 0;
          const unsigned long long a = sorted[i], bb = sorted[jx];
          if ((a < bb) == desc) { sorted[i] = bb; sorted[jx] = a; }
        }
      }
      __syncthreads();
    }
  }
  for (int i = tid; i < k; i += kSelThreads) {
    const unsigned long long key = sorted[i];
    const bool v = key != 0ull;
    idx[static_cast<size_t>(b) * k + i] = v ? static_cast<int32_t>(topk_key_index(key)) : -1;
    if (scores) scores[static_cast<size_t>(b) * k + i] = v ? order_key_to_float(static_cast<uint32_t>(key >> 32)) : -INFINITY;
  }
}

// ------------------------------------------------------------------------------------
// host side

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void *ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

bool make_rows_map(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kRowBytes), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kRowBytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kRowBytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int tc_grid() { return sm_count(); }

int64_t cand_stride(const IndexerLaunch &p) {
  const int64_t capacity = static_cast<int64_t>(p.max_blocks) * (DSV4_PAGE_POSITIONS / p.m);
  if (indexer_uses_tensor_cores(p)) {
    const int64_t tiles = (capacity + kTile - 1) / kTile;
    const int64_t lists = tiles < tc_grid() ? tiles : tc_grid();
    return (lists > 0 ? lists : 1) * p.k;
  }
  return capacity > 0 ? capacity : 1;
}

template <int H>
cudaError_t launch_tc(const IndexerLaunch &p, unsigned long long *cand, int64_t stride, int *cand_count,
                      cudaStream_t st) {
  TcParams tp;
  const int per_page = DSV4_PAGE_POSITIONS / p.m;
  const int box_rows = per_page < kTile ? per_page : kTile;
  if (!make_rows_map(&tp.tmap_k, p.k_pages, static_cast<uint64_t>(p.num_pages) * per_page, box_rows))
    return cudaErrorInvalidValue;
  if (!make_rows_map(&tp.tmap_q, p.q, static_cast<uint64_t>(p.B) * H, H)) return cudaErrorInvalidValue;
  tp.k_scales = p.k_scales;
  tp.block_table = p.block_table;
  tp.num_pages = p.num_pages;
  tp.max_blocks = p.max_blocks;
  tp.per_page = per_page;
  tp.box_rows = box_rows;
  tp.q_scale = p.q_scale;
  tp.w = p.w;
  tp.w_dt = p.w_dt;
  tp.B = p.B;
  tp.k = p.k;
  tp.m = p.m;
  tp.n_entries = p.n_entries;
  tp.pos = p.pos;
  tp.cand = cand;
  tp.stride = stride;
  tp.cand_count = cand_count;
  tp.d_status = p.d_status;
  const size_t smem = sizeof(TcSmem<H>) + 1024 + (2 * static_cast<size_t>(p.B) + 1) * 8;
  cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<H>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  indexer_tc_kernel<H><<<tc_grid(), kTcThreads, smem, st>>>(tp);
  return cudaGetLastError();
}

}  // namespace

bool indexer_uses_tensor_cores(const IndexerLaunch &p) {
  return p.k_dt == DSV4_FP8E4M3 && p.q_dt == DSV4_FP8E4M3 && p.Dq == kRowBytes &&
         (p.H == 32 || p.H == 64 || p.H == 128) && p.m <= 8 && p.k >= 1 && p.k <= kMaxK && p.q_rope_dims == 0 &&
         p.B <= 4096;
}

size_t indexer_workspace_bytes(const IndexerLaunch &p) {
  return align_up(static_cast<size_t>(p.B) * sizeof(int), 256) +
         align_up(static_cast<size_t>(p.B) * cand_stride(p) * sizeof(unsigned long long), 256);
}

cudaError_t launch_indexer_topk(const IndexerLaunch &p, void *ws, cudaStream_t st) {
  int *cand_count = static_cast<int *>(ws);
  unsigned long long *cand = reinterpret_cast<unsigned long long *>(
      static_cast<char *>(ws) + align_up(static_cast<size_t>(p.B) * sizeof(int), 256));
  const int64_t stride = cand_stride(p);
  cudaError_t e = cudaMemsetAsync(cand_count, 0, static_cast<size_t>(p.B) * sizeof(int), st);
  if (e != cudaSuccess) return e;
  if (indexer_uses_tensor_cores(p)) {
    if (p.H == 32) e = launch_tc<32>(p, cand, stride, cand_count, st);
    else if (p.H == 64) e = launch_tc<64>(p, cand, stride, cand_count, st);
    else e = launch_tc<128>(p, cand, stride, cand_count, st);
  } else {
    const int64_t capacity = static_cast<int64_t>(p.max_blocks) * (DSV4_PAGE_POSITIONS / p.m);
    dim3 grid(static_cast<unsigned>((capacity + 255) / 256), p.B);
    const size_t smem = (static_cast<size_t>(p.H) * p.Dq + p.H) * sizeof(float);
    e = cudaFuncSetAttribute(indexer_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    indexer_simt_kernel<<<grid, 256, smem, st>>>(p, cand, stride, cand_count);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) return e;
  topk_select_kernel<<<p.B, kSelThreads, 0, st>>>(cand, stride, cand_count, p.k, p.idx, p.scores, p.d_status);
  return cudaGetLastError();
}

}  // namespace dsv4
