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

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace dsv4 {

namespace {

constexpr int kTile = 128;      // entries per tile = MMA M
constexpr int kRowBytes = 128;  // fp8 key row = 128 dims
constexpr int kSelThreads = 1024;
constexpr int kMaxSortK = 2048;

// Byte histogram of the keys that match `prefix` under `mask`, one pass over keys[0, cnt)
// by `nwarps` warps. Lanes that hit the same bin are merged with match.any so a heavily
// shared bin costs one shared-memory atomic per warp instead of one per key.
__device__ __forceinline__ void hist_add_warp(int *hist, const unsigned long long *keys, int cnt, int warp,
                                              int nwarps, unsigned long long prefix, unsigned long long mask,
                                              int shift) {
  const int lane = threadIdx.x & 31;
  for (int i0 = warp * 32; i0 < cnt; i0 += nwarps * 32) {
    const int i = i0 + lane;
    int bin = 256;
    if (i < cnt) {
      const unsigned long long key = keys[i];
      if ((key & mask) == prefix) bin = static_cast<int>((key >> shift) & 0xFF);
    }
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, bin);
    if (bin < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
  }
}

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
  CUtensorMap tmap_k;  // keys as [num_pages * 64 rows][128 bytes], 128B swizzle
  CUtensorMap tmap_q;  // queries as [B * H rows][128 bytes], 128B swizzle
  const float *k_scales;
  const int32_t *block_table;
  int num_pages, max_blocks;
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

// The tensor-core path serves C4 layers: 64 entries per page, a 128-entry tile = 2 pages,
// a pipeline stage = up to 2 tiles of one sequence (32 KB of keys).
constexpr int kPerPage = 64;
constexpr int kStageTiles = 2;
constexpr int kStages = 5;       // key stages in flight (160 KB)
constexpr int kSlots = 8;        // key-scale ring, one slot per stage
constexpr int kGroups = 2;       // epilogue warp groups, alternating stages
constexpr int kCapG = 1024;      // candidate buffer of a group
constexpr int kMaxKTc = 512;     // largest k of the tensor-core path
constexpr int kGroupThreads = 128;
constexpr int kIxThreads = 64 + kGroups * kGroupThreads;

struct GroupState {
  unsigned long long thr, sel_prefix, sel_mask;
  int cnt, cnt2, out_base, sel_digit, sel_above, sel_count, stop;
};

template <int H>  // H in {32, 64}
struct alignas(1024) TcSmem {
  uint8_t stage[kStages][kStageTiles][kTile * kRowBytes];  // key tiles (rows = entries)
  uint8_t q[2][H * kRowBytes];
  float sig[kSlots][kStageTiles * kTile];                   // key scales of each stage (0: no key)
  unsigned long long cand[kGroups][kCapG];
  unsigned long long cand2[kGroups][kMaxKTc];
  float coef[kGroups][H];
  int hist[kGroups][256];
  uint64_t full[kStages], empty[kStages], sfull[kSlots], sempty[kSlots];
  uint64_t tfull[kGroups], tempty[kGroups], qfull[2], qempty[2];
  GroupState gs[kGroups];
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ int find_seq(const long long *prefix, int B, long long g) {
  int lo = 0, hi = B - 1;  // last b with prefix[b] <= g
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Walks a CTA's tile range [t0, t1) as stages of up to 2 tiles that never cross a sequence.
struct StageIter {
  long long g, t1;
  int b;
  bool first;
  __device__ void init(const long long *prefix, int B, long long t0, long long t1_) {
    g = t0;
    t1 = t1_;
    b = t0 < t1_ ? find_seq(prefix, B, t0) : 0;
    first = true;
  }
  __device__ bool next(const long long *prefix, int &sb, long long &lt0, int &nt, bool &new_seg, bool &seg_end) {
    if (g >= t1) return false;
    new_seg = first;
    first = false;
    while (g >= prefix[b + 1]) {
      ++b;
      new_seg = true;
    }
    const long long end = prefix[b + 1] < t1 ? prefix[b + 1] : t1;
    nt = end - g >= kStageTiles ? kStageTiles : static_cast<int>(end - g);
    sb = b;
    lt0 = g - prefix[b];
    g += nt;
    seg_end = g >= end;
    return true;
  }
};

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
// one arrival on bar once every earlier cp.async of this thread has landed
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Top-k of one epilogue group: MSB-first radix select over the bytes of the (distinct)
// 64-bit keys of cand[gi][0..cnt). Leaves (prefix, mask) such that
// {key : (key & mask) >= prefix} has exactly k elements. 128 threads of the group.
template <int H>
__device__ void group_select(TcSmem<H> &S, int gi, int cnt, int k, int gt) {
  GroupState &G = S.gs[gi];
  int *hist = S.hist[gi];
  const int bar = 1 + gi;
  unsigned long long prefix = 0, mask = 0;
  int need = k;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int i = gt; i < 256; i += kGroupThreads) hist[i] = 0;
    named_bar_sync(bar, kGroupThreads);
    hist_add_warp(hist, S.cand[gi], cnt, gt >> 5, kGroupThreads >> 5, prefix, mask, shift);
    named_bar_sync(bar, kGroupThreads);
    if (gt < 32) {
      int c[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) { c[u] = hist[255 - gt * 8 - u]; tot += c[u]; }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (gt >= o) incl += v;
      }
      int run = incl - tot;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (run < need && run + c[u] >= need) {
          G.sel_digit = 255 - gt * 8 - u;
          G.sel_above = run;
          G.sel_count = c[u];
        }
        run += c[u];
      }
    }
    named_bar_sync(bar, kGroupThreads);
    const int digit = G.sel_digit, above = G.sel_above, cntd = G.sel_count;
    prefix |= static_cast<unsigned long long>(digit) << shift;
    mask |= 0xFFull << shift;
    need -= above;
    named_bar_sync(bar, kGroupThreads);
    if (cntd == need) break;
  }
  if (gt == 0) { G.sel_prefix = prefix; G.sel_mask = mask; }
  named_bar_sync(bar, kGroupThreads);
}

// keep exactly the k best candidates of group gi and raise its insertion threshold
template <int H>
__device__ void group_compact(TcSmem<H> &S, int gi, int k, int gt) {
  GroupState &G = S.gs[gi];
  const int bar = 1 + gi;
  const int cnt = G.cnt;
  group_select(S, gi, cnt, k, gt);
  const unsigned long long prefix = G.sel_prefix, mask = G.sel_mask;
  if (gt == 0) G.cnt2 = 0;
  named_bar_sync(bar, kGroupThreads);
  for (int i = gt; i < cnt; i += kGroupThreads) {
    const unsigned long long key = S.cand[gi][i];
    if ((key & mask) >= prefix) {
      const int at = atomicAdd(&G.cnt2, 1);
      if (at < kMaxKTc) S.cand2[gi][at] = key;
    }
  }
  named_bar_sync(bar, kGroupThreads);
  const int kept = G.cnt2 < k ? G.cnt2 : k;
  for (int i = gt; i < kept; i += kGroupThreads) S.cand[gi][i] = S.cand2[gi][i];
  named_bar_sync(bar, kGroupThreads);
  if (gt == 0) {
    G.cnt = kept;
    if (prefix > G.thr) G.thr = prefix;
  }
  named_bar_sync(bar, kGroupThreads);
}

template <int H>
__device__ void group_flush(TcSmem<H> &S, const TcParams &p, int gi, int b, int gt) {
  GroupState &G = S.gs[gi];
  const int bar = 1 + gi;
  named_bar_sync(bar, kGroupThreads);
  if (G.cnt > p.k) group_compact(S, gi, p.k, gt);
  const int nout = G.cnt;
  if (gt == 0) G.out_base = atomicAdd(&p.cand_count[b], nout);
  named_bar_sync(bar, kGroupThreads);
  const int base = G.out_base;
  if (base + nout > p.stride) {
    if (gt == 0) report(p.d_status, DSV4_DEV_BAD_LENGTH);
  } else {
    for (int i = gt; i < nout; i += kGroupThreads) p.cand[static_cast<size_t>(b) * p.stride + base + i] = S.cand[gi][i];
  }
  named_bar_sync(bar, kGroupThreads);
}

template <int H>
__global__ void __launch_bounds__(kIxThreads, 1) indexer_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem<H> &S = *reinterpret_cast<TcSmem<H> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  long long *prefix = reinterpret_cast<long long *>(&S + 1);       // [B + 1] tiles before sequence b
  int64_t *nvis = reinterpret_cast<int64_t *>(prefix + p.B + 1);  // [B] visible entries
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t capacity = static_cast<int64_t>(p.max_blocks) * kPerPage;

  // ---- setup: barriers, TMEM, tile prefix over sequences
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], 1); }
    for (int i = 0; i < kSlots; ++i) { mbar_init(&S.sfull[i], 32); mbar_init(&S.sempty[i], kGroupThreads / 32); }
    for (int i = 0; i < kGroups; ++i) { mbar_init(&S.tfull[i], 1); mbar_init(&S.tempty[i], kGroupThreads / 32); }
    for (int i = 0; i < 2; ++i) { mbar_init(&S.qfull[i], 1); mbar_init(&S.qempty[i], 1); }
    S.abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tmap_k);
    prefetch_tensormap(&p.tmap_q);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kGroups * kStageTiles * H);
    tmem_relinquish();
  }
  for (int b = tid; b < p.B; b += kIxThreads)
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
    // ---------------- producer. Lane 0 issues the key TMA of stage k; the 32 lanes copy
    // the key scales of stage k into scale slot k % kSlots with cp.async (two 16-byte copies
    // per lane), each lane's copies arriving on the slot's barrier when they land, so
    // neither the block-table nor the scale latency stalls the key stream.
    // Page ids of stage k+1 are fetched while stage k is issued. A page that is invalid
    // or starts past the visible entries gets scale 0 and a zero-filled key box.
    const int oob_row = p.num_pages * kPerPage;
    StageIter it, ahead;
    it.init(prefix, p.B, t0, t1);
    ahead = it;
    int ab, ant;
    long long alt0;
    bool anew, aend;
    // page id of this lane's page in the next stage (lanes 0..3)
    auto fetch_pid = [&](int sb, long long lt0, int nt) -> int {
      int pid = -1;
      if (lane < nt * kStageTiles) {
        const int64_t first = lt0 * kTile + static_cast<int64_t>(lane) * kPerPage;
        if (first < nvis[sb]) {
          const int pg = p.block_table[static_cast<size_t>(sb) * p.max_blocks + first / kPerPage];
          if (pg >= 0 && pg < p.num_pages) pid = pg;
          else report(p.d_status, DSV4_DEV_BAD_PAGE);
        }
      }
      return pid;
    };
    int pid_next = -1;
    if (ahead.next(prefix, ab, alt0, ant, anew, aend)) pid_next = fetch_pid(ab, alt0, ant);
    int seg = -1;
    long long k = 0;
    bool stop = false;
    int sb, nt;
    long long lt0;
    bool new_seg, seg_end;
    while (!stop && it.next(prefix, sb, lt0, nt, new_seg, seg_end)) {
      const int pid = pid_next;
      pid_next = -1;
      if (ahead.next(prefix, ab, alt0, ant, anew, aend)) pid_next = fetch_pid(ab, alt0, ant);
      const int slot = static_cast<int>(k % kSlots);
      int ok = 1;
      if (lane == 0 && k >= kSlots &&
          !mbar_wait(&S.sempty[slot], static_cast<uint32_t>((k / kSlots - 1) & 1), &S.abort_flag))
        ok = 0;
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      {  // scales of stage k: lane l copies 2 x 16 bytes of page l / 8
        const int pg_slot = lane >> 3;  // 0..3 = tile * 2 + half
        const int my_pid = __shfl_sync(0xFFFFFFFFu, pid, pg_slot);
        float *dst = &S.sig[slot][pg_slot * kPerPage + (lane & 7) * 8];
        if (my_pid >= 0) {
          const float *src = p.k_scales + static_cast<size_t>(my_pid) * kPerPage + (lane & 7) * 8;
          cp_async16(dst, src);
          cp_async16(dst + 4, src + 4);
          cp_async_arrive(&S.sfull[slot]);
        } else {
          reinterpret_cast<float4 *>(dst)[0] = make_float4(0.f, 0.f, 0.f, 0.f);
          reinterpret_cast<float4 *>(dst)[1] = make_float4(0.f, 0.f, 0.f, 0.f);
          mbar_arrive(&S.sfull[slot]);
        }
      }
      int rows[kStageTiles * 2];
#pragma unroll
      for (int i = 0; i < kStageTiles * 2; ++i) {
        const int v = __shfl_sync(0xFFFFFFFFu, pid, i);
        rows[i] = v >= 0 ? v * kPerPage : oob_row;
      }
      if (lane == 0) {
        if (new_seg) {
          ++seg;
          const int qs = seg & 1;
          if (seg >= 2 && !mbar_wait(&S.qempty[qs], ((seg >> 1) - 1) & 1, &S.abort_flag)) ok = 0;
          if (ok) {
            mbar_arrive_expect_tx(&S.qfull[qs], H * kRowBytes);
            tma_load_2d(S.q[qs], &p.tmap_q, &S.qfull[qs], 0, sb * H);
          }
        }
        const int s = static_cast<int>(k % kStages);
        if (ok && k >= kStages && !mbar_wait(&S.empty[s], static_cast<uint32_t>((k / kStages - 1) & 1), &S.abort_flag))
          ok = 0;
        if (ok) {
          mbar_arrive_expect_tx(&S.full[s], static_cast<uint32_t>(nt) * kTile * kRowBytes);
          for (int t = 0; t < nt; ++t)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tma_load_2d(S.stage[s][t] + h * kPerPage * kRowBytes, &p.tmap_k, &S.full[s], 0, rows[t * 2 + h]);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) {
        stop = true;
        break;
      }
      ++k;
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    if (lane == 0 && S.abort_flag) {
      // let key loads already in flight land before the CTA leaves
      const long long from = k > kStages ? k - kStages : 0;
      for (long long n = from; n < k; ++n) {
        volatile int dummy = 0;
        mbar_wait(&S.full[n % kStages], static_cast<uint32_t>((n / kStages) & 1), &dummy);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: stage k goes to accumulator set k % 2 (read by group k % 2)
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3(kTile, H);
      StageIter it;
      it.init(prefix, p.B, t0, t1);
      int sb, nt, seg = -1;
      long long lt0, k = 0;
      bool new_seg, seg_end;
      while (it.next(prefix, sb, lt0, nt, new_seg, seg_end)) {
        if (new_seg) {
          ++seg;
          if (!mbar_wait(&S.qfull[seg & 1], (seg >> 1) & 1, &S.abort_flag)) break;
        }
        const int s = static_cast<int>(k % kStages);
        if (!mbar_wait(&S.full[s], static_cast<uint32_t>((k / kStages) & 1), &S.abort_flag)) break;
        const int a = static_cast<int>(k % kGroups);
        if (k >= kGroups && !mbar_wait(&S.tempty[a], static_cast<uint32_t>((k / kGroups - 1) & 1), &S.abort_flag)) break;
        tc_fence_after();
        const uint32_t b0 = smem_u32(S.q[seg & 1]);
        for (int t = 0; t < nt; ++t) {
          const uint32_t a0 = smem_u32(S.stage[s][t]);
#pragma unroll
          for (int kk = 0; kk < kRowBytes / 32; ++kk)
            mma_e4m3(tmem + (a * kStageTiles + t) * H, sw128_desc(a0 + kk * 32, 16, 1024),
                     sw128_desc(b0 + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&S.empty[s]);
        mma_commit(&S.tfull[a]);
        if (seg_end) mma_commit(&S.qempty[seg & 1]);
        ++k;
      }
    }
  } else {
    // ---------------- epilogue groups (warps 2..5: group 0, warps 6..9: group 1). Group gi
    // scores the stages k with k % 2 == gi and keeps its own running top-k per sequence.
    const int gi = (warp - 2) / 4;
    const int gt = tid - 64 - gi * kGroupThreads;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int bar = 1 + gi;
    GroupState &GS = S.gs[gi];
    StageIter it;
    it.init(prefix, p.B, t0, t1);
    int sb, nt, cur_b = -1;
    long long lt0, k = 0;
    bool new_seg, seg_end;
    unsigned long long thr = 1;
    while (it.next(prefix, sb, lt0, nt, new_seg, seg_end)) {
      const long long kk = k++;
      if (kk % kGroups != gi) continue;
      if (sb != cur_b) {
        if (cur_b >= 0) group_flush(S, p, gi, cur_b, gt);
        cur_b = sb;
        for (int h = gt; h < H; h += kGroupThreads) {
          const float qs = p.q_scale ? p.q_scale[static_cast<size_t>(sb) * H + h] : 1.0f;
          S.coef[gi][h] = load_one_f(p.w, p.w_dt, static_cast<size_t>(sb) * H + h) * qs;
        }
        if (gt == 0) { GS.cnt = 0; GS.thr = 1; }
        thr = 1;
        named_bar_sync(bar, kGroupThreads);
      }
      const int slot = static_cast<int>(kk % kSlots);
      bool ok = mbar_wait(&S.sfull[slot], static_cast<uint32_t>((kk / kSlots) & 1), &S.abort_flag);
      ok = mbar_wait(&S.tfull[gi], static_cast<uint32_t>((kk / kGroups) & 1), &S.abort_flag) && ok;
      ok = __all_sync(0xFFFFFFFFu, ok);
      unsigned long long key[kStageTiles] = {0ull, 0ull};
      if (ok) {
        tc_fence_after();
        const float4 *cf4 = reinterpret_cast<const float4 *>(S.coef[gi]);
        // one tile at a time keeps 64 accumulator registers live, not 128
#pragma unroll
        for (int t = 0; t < kStageTiles; ++t) {
          if (t < nt) {
            uint32_t r[H];
            const uint32_t ta = tmem + (static_cast<uint32_t>(quad * 32) << 16) + (gi * kStageTiles + t) * H;
            tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
            if (H > 32) tmem_ld32(ta + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32 % H]));
            const float sc = S.sig[slot][t * kTile + row];
            tmem_ld_wait();
            float part[4] = {0.f, 0.f, 0.f, 0.f};  // 4 short chains, not one of H
#pragma unroll
            for (int i = 0; i < H; i += 4) {
              const float4 c = cf4[i / 4];
              part[0] = fmaf(c.x, fmaxf(__uint_as_float(r[i]), 0.f), part[0]);
              part[1] = fmaf(c.y, fmaxf(__uint_as_float(r[i + 1]), 0.f), part[1]);
              part[2] = fmaf(c.z, fmaxf(__uint_as_float(r[i + 2]), 0.f), part[2]);
              part[3] = fmaf(c.w, fmaxf(__uint_as_float(r[i + 3]), 0.f), part[3]);
            }
            const float score = ((part[0] + part[1]) + (part[2] + part[3])) * sc;
            const int64_t j = (lt0 + t) * kTile + row;
            if (j < nvis[sb] && sc > 0.f) key[t] = topk_key(score, static_cast<uint32_t>(j));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&S.tempty[gi]);
          mbar_arrive(&S.sempty[slot]);
        }
      } else if (lane == 0) {
        S.abort_flag = 1;
      }
      // insert the keys that beat the group's threshold
#pragma unroll
      for (int t = 0; t < kStageTiles; ++t) {
        const bool pass = key[t] != 0ull && key[t] >= thr;
        const unsigned bal = __ballot_sync(0xFFFFFFFFu, pass);
        int base = 0;
        if (lane == 0 && bal) base = atomicAdd(&GS.cnt, __popc(bal));
        base = __shfl_sync(0xFFFFFFFFu, base, 0);
        if (pass) S.cand[gi][base + __popc(bal & ((1u << lane) - 1u))] = key[t];
      }
      // one group barrier per stage: abort check, and compaction when the buffer could
      // not take another stage (abort_flag is read after the barrier by every warp)
      named_bar_sync(bar, kGroupThreads);
      if (gt == 0) GS.stop = S.abort_flag;
      named_bar_sync(bar, kGroupThreads);
      if (GS.stop) break;
      if (GS.cnt > kCapG - kStageTiles * kTile) group_compact(S, gi, p.k, gt);
      thr = GS.thr;
    }
    if (cur_b >= 0 && !GS.stop) group_flush(S, p, gi, cur_b, gt);
  }

  if (tid == 0 && S.abort_flag) report(p.d_status, DSV4_DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kGroups * kStageTiles * H);
  }
}

// ------------------------------------------------------------------------------------
// Per-sequence select: the k best keys of the candidate list, sorted (score desc,
// index asc), written as entry indices (+ scores); -1 / -inf padding.

__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(const unsigned long long *cand, int64_t stride,
                                                                  const int *cand_count, int k, int32_t *idx,
                                                                  float *scores, uint32_t *d_status, int smem_keys) {
  extern __shared__ unsigned long long skeys[];  // [smem_keys] staged candidates, then [kp2] selected
  __shared__ int hist[256];
  __shared__ int sel_digit, sel_above, sel_count, kept;
  const int b = blockIdx.x, tid = threadIdx.x;
  const unsigned long long *c = cand + static_cast<size_t>(b) * stride;
  int cnt = cand_count[b];
  if (cnt > stride) {
    if (tid == 0) report(d_status, DSV4_DEV_BAD_LENGTH);
    cnt = static_cast<int>(stride);
  }
  int kp2 = 1;
  while (kp2 < k) kp2 <<= 1;
  // candidates in shared memory when they fit next to the kp2 output slots
  const bool staged = cnt + kp2 <= smem_keys;
  unsigned long long *sorted = skeys + (staged ? cnt : 0);
  if (staged) {
    for (int i = tid; i < cnt; i += kSelThreads) skeys[i] = c[i];
    c = skeys;
  }
  __syncthreads();
  unsigned long long prefix = 0, mask = 0;
  if (cnt > k) {
    int need = k;
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      hist_add_warp(hist, c, cnt, tid >> 5, kSelThreads >> 5, prefix, mask, shift);
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
  // bitonic sort, descending: output order (score desc, index asc) does not depend on timing
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
    // one list of at most k keys per (CTA, epilogue group) that touches the sequence
    const int64_t tiles = (capacity + kTile - 1) / kTile;
    const int64_t ctas = tiles < tc_grid() ? tiles : tc_grid();
    return (ctas > 0 ? ctas : 1) * kGroups * p.k;
  }
  return capacity > 0 ? capacity : 1;
}

template <int H>
cudaError_t launch_tc(const IndexerLaunch &p, unsigned long long *cand, int64_t stride, int *cand_count,
                      cudaStream_t st) {
  TcParams tp;
  if (!make_rows_map(&tp.tmap_k, p.k_pages, static_cast<uint64_t>(p.num_pages) * kPerPage, kPerPage))
    return cudaErrorInvalidValue;
  if (!make_rows_map(&tp.tmap_q, p.q, static_cast<uint64_t>(p.B) * H, H)) return cudaErrorInvalidValue;
  tp.k_scales = p.k_scales;
  tp.block_table = p.block_table;
  tp.num_pages = p.num_pages;
  tp.max_blocks = p.max_blocks;
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
  indexer_tc_kernel<H><<<tc_grid(), kIxThreads, smem, st>>>(tp);
  return cudaGetLastError();
}

}  // namespace

bool indexer_uses_tensor_cores(const IndexerLaunch &p) {
  return p.k_dt == DSV4_FP8E4M3 && p.q_dt == DSV4_FP8E4M3 && p.Dq == kRowBytes &&
         (p.H == 32 || p.H == 64) && p.m == 4 && p.k >= 1 && p.k <= kMaxKTc && p.q_rope_dims == 0 &&
         p.B <= 512;
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
    else e = launch_tc<64>(p, cand, stride, cand_count, st);
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
  // stage up to ~200 KB of candidates in shared memory (the rest of the kernel's smem is small)
  const int smem_keys = static_cast<int>(std::min<int64_t>(stride + kMaxSortK, 25600));
  const size_t ssmem = static_cast<size_t>(smem_keys) * sizeof(unsigned long long);
  e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
  if (e != cudaSuccess) return e;
  topk_select_kernel<<<p.B, kSelThreads, ssmem, st>>>(cand, stride, cand_count, p.k, p.idx, p.scores, p.d_status,
                                                      smem_keys);
  return cudaGetLastError();
}

}  // namespace dsv4
