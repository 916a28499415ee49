// Lightning indexer + top-k (step (2) of the decode method; "DeepSeek Sparse Attention
// over compressed tokens" in the vLLM post, "Lightning TopK" in the SGLang blog).
//
//   s_j = sum_h w_h * ReLU(q_h . k_j)       for every visible C4 entry j
//   keep the k largest s_j (ties to the lower j)
//
// Tensor-core path (fp8 or fp4 keys, 128-dim, the C4 layers): a persistent kernel, one CTA
// per SM, over the flattened (sequence, 128-entry tile) space, in stages of up to four tiles
// of one sequence. Warp 0 streams key pages with TMA (one 64-row box per page and lane,
// 128B swizzle) into a ring of 2 or 3 stages of 64 KB, with the block-table entries fetched
// a batch of 4 stages ahead, and hands each stage's page rows to the epilogue; warp 1 issues
// tcgen05.mma kind::f8f6f4 (M = 128 entries, N = H heads, K = 128) into two TMEM accumulator
// sets; two groups of four warps take alternate stages, load their keys' scales, read their
// accumulators back (tcgen05.ld), apply ReLU, the per-head weights w_h * scale_q[h] and the
// per-entry key scale, and store every score (4 bytes per entry, coalesced). A second kernel selects the
// top k of each sequence from the scores (a cluster radix select over registers), writing
// them in ascending entry order.
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

// Entries of sequence b the selection sees: n_entries[b], or (without it) the complete blocks
// once the token at pos[b] is in, floor((pos + 1) / m); `appended` = 0 counts them before that
// token's append, floor(pos / m).
__device__ __forceinline__ int64_t visible_entries(const int32_t *n_entries, const int32_t *pos, int m, int b,
                                                   int64_t capacity, uint32_t *d_status, bool report_it,
                                                   int appended = 1) {
  int64_t n = n_entries ? static_cast<int64_t>(n_entries[b]) : (static_cast<int64_t>(pos[b]) + appended) / m;
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
  pdl_wait();
  pdl_launch_dependents();
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
      rope_cos_sin(p.pos[b], i, p.rope_theta1, &c, &s);
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
    const float ks = (p.k_dt == DSV4_FP8E4M3 || p.k_dt == DSV4_FP4E2M1) ? p.k_scales[row] : 1.0f;
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
// Tensor-core scoring: every visible entry's score streamed to a [B][ld] float buffer.

struct TcParams {
  CUtensorMap tmap_k;  // keys as [num_pages * 64 rows][128 bytes], 128B swizzle
  CUtensorMap tmap_q;  // queries as [B * H rows][128 bytes], 128B swizzle
  const float *k_scales;
  const int32_t *block_table;
  int num_pages, max_blocks;
  const float *q_scale;
  const void *w;
  dsv4_dtype w_dt;
  int B, m;
  const int32_t *n_entries;
  const int32_t *pos;
  float *scores;  // [B][ld]; -inf where the entry has no valid page
  int64_t ld;
  uint32_t *d_status;
  int before_append;  // score only the entries visible before this step's append (floor(pos / m))
  int keys_fp4;       // keys are e2m1 (64 bytes per row in global memory) instead of e4m3
  int release;  // release the next kernel early (always: the top-k kernel follows)
};

// The tensor-core path serves C4 layers: 64 entries per page, a 128-entry tile = 2 pages,
// a pipeline stage = up to 4 tiles of one sequence (64 KB of keys in shared memory). Larger
// stages halve the producer's per-stage bookkeeping per byte, which had set its pace.
constexpr int kPerPage = 64;
constexpr int kStageTiles = 4;
constexpr int kStagePages = kStageTiles * kTile / kPerPage;
constexpr int kStagesHi = 12 / kStageTiles;  // 192 KB of key stages in flight, or one stage less
constexpr int kStagesLo = kStagesHi - 1;
constexpr int kSlots = 8;        // ring of the stages' page rows, one slot per stage
constexpr int kBatchStages = 32 / kStagePages;  // stages whose page ids one warp load covers (4)
constexpr int kGroups = 2;       // epilogue warp groups, alternating stages
constexpr int kGroupThreads = 128;
constexpr int kIxThreads = 64 + kGroups * kGroupThreads;

template <int H, int kStages>  // H in {32, 64}; kStages key stages of 64 KB in flight
struct alignas(1024) TcSmem {
  uint8_t stage[kStages][kStageTiles][kTile * kRowBytes];  // key tiles (rows = entries)
  uint8_t q[2][H * kRowBytes];
  int spage[kSlots][kStagePages];          // first key-scale row of each page of a stage (or past the pool: none)
  float coef[kGroups * 4][H];              // per epilogue warp: w_h * scale_q[h] of its sequence
  uint64_t full[kStages], empty[kStages], sfull[kSlots], sempty[kSlots];
  uint64_t tfull[kGroups], tempty[kGroups], qfull[2], qempty[2];
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

// Walks a CTA's tile range [t0, t1) as stages of up to kStageTiles tiles that never cross a sequence.
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

// Block-table entries of the next kBatchStages stages, one per lane (lane = kStagePages *
// stage + page): the loads of a whole batch are in flight together, a batch ahead of their use.
// Returns the raw entry (the load is not waited for here: the address is always valid and
// nothing reads the value until the batch is used) and whether the lane's slot has a page.
struct PageBatch {
  int raw;
  bool has;
  // the entry, or -1 (no page); the first read of `raw`, so the wait for its load is here
  __device__ __forceinline__ int get() const { return has ? raw : -1; }
};

__device__ __forceinline__ PageBatch load_page_batch(const TcParams &p, const long long *prefix, const int64_t *nvis,
                                                     StageIter &ahead, int lane) {
  int sb_l = -1;
  int64_t first_l = 0;
#pragma unroll 1
  for (int i = 0; i < kBatchStages; ++i) {
    int sb, nt;
    long long lt0;
    bool ns, se;
    if (!ahead.next(prefix, sb, lt0, nt, ns, se)) break;
    if (lane / kStagePages == i && lane % kStagePages < nt * (kTile / kPerPage)) {
      sb_l = sb;
      first_l = lt0 * kTile + static_cast<int64_t>(lane % kStagePages) * kPerPage;
    }
  }
  // no page when the slot has no tile or starts past the visible entries; the entry is
  // validated where it is used
  PageBatch r;
  r.has = sb_l >= 0 && first_l < nvis[sb_l];
  r.raw = p.block_table[r.has ? static_cast<size_t>(sb_l) * p.max_blocks + first_l / kPerPage : 0];
  return r;
}

template <int H, int kStages>
__global__ void __launch_bounds__(kIxThreads, 1) indexer_tc_kernel(const __grid_constant__ TcParams p) {
  extern __shared__ uint8_t smem_raw[];
  TcSmem<H, kStages> &S =
      *reinterpret_cast<TcSmem<H, kStages> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  long long *prefix = reinterpret_cast<long long *>(&S + 1);       // [B + 1] tiles before sequence b
  int64_t *nvis = reinterpret_cast<int64_t *>(prefix + p.B + 1);  // [B] visible entries
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t capacity = static_cast<int64_t>(p.max_blocks) * kPerPage;

  // ---- setup: barriers, TMEM, tile prefix over sequences
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) { mbar_init(&S.full[i], 1); mbar_init(&S.empty[i], 1); }
    for (int i = 0; i < kSlots; ++i) { mbar_init(&S.sfull[i], kStagePages); mbar_init(&S.sempty[i], kGroupThreads / 32); }
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
    nvis[b] = visible_entries(p.n_entries, p.pos, p.m, b, capacity, p.d_status, blockIdx.x == 0,
                              p.before_append ? 0 : 1);
  __syncthreads();
  StageIter it, ahead;                // the producer's walk over its stages (warp 0)
  PageBatch batch_cur{}, batch_next{};  // and its first two batches of page ids
  if (warp == 0) {  // tiles per sequence, scanned by one warp
    long long carry = 0;
    for (int b0 = 0; b0 < p.B; b0 += 32) {
      const int b = b0 + lane;
      const long long c = b < p.B ? (nvis[b] + kTile - 1) / kTile : 0;
      long long v = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if (lane >= o) v += u;
      }
      if (b < p.B) prefix[b] = carry + v - c;
      carry += __shfl_sync(0xFFFFFFFFu, v, 31);
    }
    if (lane == 0) prefix[p.B] = carry;
    __syncwarp();
    // The block table is written by none of the library's kernels (the only ones that may
    // still run when this one starts early), so its first two batches load before the wait.
    const long long G = gridDim.x;
    it.init(prefix, p.B, (carry * blockIdx.x) / G, (carry * (blockIdx.x + 1)) / G);
    ahead = it;
    batch_cur = load_page_batch(p, prefix, nvis, ahead, lane);
    batch_next = load_page_batch(p, prefix, nvis, ahead, lane);
  }
  // Keys and scales may be written by the kernel before: every read waits for it. (In a
  // decode step this kernel runs first, beside the step's own updates, which touch no entry it
  // scores.)
  pdl_wait();
  if (p.release) pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const long long T = prefix[p.B];
  const long long G = gridDim.x;
  const long long t0 = (T * blockIdx.x) / G, t1 = (T * (blockIdx.x + 1)) / G;

  if (warp == 0) {
    // ---------------- producer. Per stage, lanes 0..7 take one 64-row page each: its page
    // row goes to a small ring for the epilogue (which loads the keys' scales itself), and
    // its key box is issued as one TMA (an invalid page, or one past the visible entries,
    // takes a zero-filled out-of-range box), completing as transaction bytes on the stage's
    // barrier. Ring positions and phases are kept as counters: no division in the loop.
    const int oob_row = p.num_pages * kPerPage;
    int seg = -1;
    int k = 0, bs = 0;              // stage count; stage within the page batch
    int s = 0, slot = 0;            // key ring stage and page-row slot
    uint32_t s_lap = 0, slot_lap = 0;
    int sb, nt;
    long long lt0;
    bool new_seg, seg_end;
    while (it.next(prefix, sb, lt0, nt, new_seg, seg_end)) {
      if (bs == kBatchStages) {
        bs = 0;
        batch_cur = batch_next;
        batch_next = load_page_batch(p, prefix, nvis, ahead, lane);
      }
      // this lane's page (lanes 0..7), validated: an entry outside the pool is reported and
      // treated as no page
      int pid = __shfl_sync(0xFFFFFFFFu, batch_cur.get(), (bs * kStagePages + lane) & 31);
      if (lane < kStagePages && pid != -1 && (pid < 0 || pid >= p.num_pages)) {
        report(p.d_status, DSV4_DEV_BAD_PAGE);
        pid = -1;
      }
      const int row = pid >= 0 ? pid * kPerPage : oob_row;
      int ok = 1;
      if (lane < kStagePages) {
        if (k >= kSlots && !mbar_wait(&S.sempty[slot], (slot_lap - 1) & 1, &S.abort_flag)) ok = 0;
        if (ok) {
          S.spage[slot][lane] = row;
          mbar_arrive(&S.sfull[slot]);
        }
      }
      if (lane == 0) {
        if (ok && new_seg) {
          ++seg;
          const int qs = seg & 1;
          if (seg >= 2 && !mbar_wait(&S.qempty[qs], ((seg >> 1) - 1) & 1, &S.abort_flag)) ok = 0;
          if (ok) {
            mbar_arrive_expect_tx(&S.qfull[qs], H * kRowBytes);
            tma_load_2d(S.q[qs], &p.tmap_q, &S.qfull[qs], 0, sb * H);
          }
        }
        if (ok && k >= kStages && !mbar_wait(&S.empty[s], (s_lap - 1) & 1, &S.abort_flag)) ok = 0;
        // (fp4 keys: the transaction counts the packed bytes read, half the tile)
        if (ok) mbar_arrive_expect_tx(&S.full[s], static_cast<uint32_t>(nt) * kTile * (p.keys_fp4 ? kRowBytes / 2 : kRowBytes));
      }
      ok = __all_sync(0xFFFFFFFFu, ok);
      if (!ok) break;
      if (lane < nt * (kTile / kPerPage))  // lane i: page i % 2 of tile i / 2
        tma_load_2d(S.stage[s][lane >> 1] + (lane & 1) * kPerPage * kRowBytes, &p.tmap_k, &S.full[s], 0, row);
      ++k;
      ++bs;
      if (++s == kStages) { s = 0; ++s_lap; }
      if (++slot == kSlots) { slot = 0; ++slot_lap; }
    }
    if (lane == 0 && S.abort_flag) {
      // let key loads already in flight land before the CTA leaves: the stages issued, the
      // last kStages of them (stage k - n sits at ring position s - n)
      const int from = k > kStages ? kStages : k;
      for (int n = from; n >= 1; --n) {
        const int q = k - n;
        volatile int dummy = 0;
        mbar_wait(&S.full[q % kStages], static_cast<uint32_t>((q / kStages) & 1), &dummy);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: stage k goes to accumulator set k % 2 (read by group k % 2)
    if (lane == 0) {
      const uint32_t idesc = p.keys_fp4 ? idesc_e2m1_e4m3(kTile, H) : idesc_e4m3(kTile, H);
      StageIter it;
      it.init(prefix, p.B, t0, t1);
      int sb, nt, seg = -1;
      long long lt0;
      int k = 0, s = 0;
      uint32_t s_lap = 0;
      bool new_seg, seg_end;
      while (it.next(prefix, sb, lt0, nt, new_seg, seg_end)) {
        if (new_seg) {
          ++seg;
          if (!mbar_wait(&S.qfull[seg & 1], (seg >> 1) & 1, &S.abort_flag)) break;
        }
        if (!mbar_wait(&S.full[s], s_lap & 1, &S.abort_flag)) break;
        const int a = k & (kGroups - 1);
        if (k >= kGroups && !mbar_wait(&S.tempty[a], static_cast<uint32_t>((k / kGroups - 1) & 1), &S.abort_flag)) break;
        tc_fence_after();
        const uint64_t bq = sw128_desc(smem_u32(S.q[seg & 1]), 16, 1024);
        for (int t = 0; t < nt; ++t) {
          const uint64_t ak = sw128_desc(smem_u32(S.stage[s][t]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kRowBytes / 32; ++kk)  // K step of 32 bytes = +2 in the descriptor
            mma_e4m3(tmem + (a * kStageTiles + t) * H, ak + 2 * kk, bq + 2 * kk, idesc, kk > 0 ? 1u : 0u);
        }
        mma_commit(&S.empty[s]);
        mma_commit(&S.tfull[a]);
        if (seg_end) mma_commit(&S.qempty[seg & 1]);
        ++k;
        if (++s == kStages) { s = 0; ++s_lap; }
      }
    }
  } else {
    // ---------------- epilogue groups (warps 2..5: group 0, warps 6..9: group 1). Group gi
    // scores the stages k with k % 2 == gi: each thread one entry row, the H accumulators
    // of its row weighted by c_h = w_h * scale_q[h] after ReLU, times the key's scale.
    const int gi = (warp - 2) / 4;
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const int oob_row = p.num_pages * kPerPage;  // (a page past the pool: no key)
    float *coef = S.coef[warp - 2];
    StageIter it;
    it.init(prefix, p.B, t0, t1);
    int sb, nt, cur_b = -1;
    long long lt0, k = 0;
    bool new_seg, seg_end;
    while (it.next(prefix, sb, lt0, nt, new_seg, seg_end)) {
      const long long kk = k++;
      if (kk % kGroups != gi) continue;
      if (sb != cur_b) {  // this warp's own copy of the sequence's head coefficients
        cur_b = sb;
        __syncwarp();
        for (int h = lane; h < H; h += 32) {
          const float qs = p.q_scale ? p.q_scale[static_cast<size_t>(sb) * H + h] : 1.0f;
          coef[h] = load_one_f(p.w, p.w_dt, static_cast<size_t>(sb) * H + h) * qs;
        }
        __syncwarp();
      }
      const int slot = static_cast<int>(kk % kSlots);
      bool ok = mbar_wait(&S.sfull[slot], static_cast<uint32_t>((kk / kSlots) & 1), &S.abort_flag);
      // this thread's key scales (0: no key), in flight while the MMA finishes
      float scl[kStageTiles];
#pragma unroll
      for (int t = 0; t < kStageTiles; ++t) {
        const int base = ok ? S.spage[slot][t * (kTile / kPerPage) + row / kPerPage] : oob_row;
        // (a coherent L2 load, not the read-only path: after a decode-step append the last
        // stage's scale was written by the kernel this one overlaps)
        scl[t] = (t < nt && base != oob_row) ? __ldcg(p.k_scales + static_cast<size_t>(base) + row % kPerPage) : 0.f;
      }
      ok = mbar_wait(&S.tfull[gi], static_cast<uint32_t>((kk / kGroups) & 1), &S.abort_flag) && ok;
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        if (lane == 0) S.abort_flag = 1;
        break;
      }
      tc_fence_after();
      float score[kStageTiles];
      const float4 *cf4 = reinterpret_cast<const float4 *>(coef);
#pragma unroll
      for (int t = 0; t < kStageTiles; ++t) {
        score[t] = -INFINITY;
        if (t < nt) {
          uint32_t r[H];
          const uint32_t ta = tmem + (static_cast<uint32_t>(quad * 32) << 16) + (gi * kStageTiles + t) * H;
          tmem_ld32(ta, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          if (H > 32) tmem_ld32(ta + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32 % H]));
          const float sc = scl[t];
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
          if (sc > 0.f) score[t] = ((part[0] + part[1]) + (part[2] + part[3])) * sc;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&S.tempty[gi]);
        mbar_arrive(&S.sempty[slot]);
      }
      const int64_t nv = nvis[sb];
      float *out = p.scores + static_cast<size_t>(sb) * p.ld;
#pragma unroll
      for (int t = 0; t < kStageTiles; ++t) {
        const int64_t j = (lt0 + t) * kTile + row;
        if (t < nt && j < nv) out[j] = score[t];
      }
    }
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
// Top-k over the score buffer: one thread-block cluster of cs CTAs per sequence, CTA r
// holding entries [r * slice, (r + 1) * slice) in shared memory as order-preserving keys
// (0 = not a candidate). An MSB-first byte radix select finds the k-th largest key with
// the cluster's histograms summed through distributed shared memory; kept are the keys
// above its class and, of the class, the lowest indices. Each warp walks a contiguous
// segment of the slice 32 keys at a time, so ballots give every kept key its rank in index
// order, and per-CTA counts exchanged in the cluster give each slice its offset: the
// output is in ascending entry order and does not depend on thread timing.

constexpr int kTkThreads = 1024;
constexpr int kTkSlice = 24 * kTkThreads;  // largest slice of a cluster CTA: 24 keys per thread
constexpr int kTkSolo = 16 * 1024;         // largest sequence one CTA takes alone (1024 threads x 16 keys)
constexpr int kTkMaxCluster = 16;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// every thread of every CTA of the cluster; orders shared-memory writes before it with reads after it
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// a shared int of CTA `rank` of this cluster
__device__ __forceinline__ int ld_cluster(const int *p, uint32_t rank) {
  uint32_t ra;
  int v;
  asm("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("ld.shared::cluster.s32 %0, [%1];" : "=r"(v) : "r"(ra));
  return v;
}
__device__ __forceinline__ int warp_sum_int(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Where the top-k kernels write: the selected entry indices (and scores).
struct TopkOut {
  int32_t *idx;        // [B][k]
  float *scores;       // [B][k] or null
  int k;
  uint32_t *d_status;

  __device__ __forceinline__ void put(int b, int o, int32_t j, float score) const {
    const size_t at = static_cast<size_t>(b) * k + o;
    idx[at] = j;
    if (scores) scores[at] = score;
  }
};

// The entry a decode step appends (entry floor((pos + 1) / m) - 1, when the step completes a
// block), scored by the top-k kernel from the cache row the step's prologue wrote, after the
// scoring kernel (which ran beside the prologue) scored the entries before it. The arithmetic
// follows the scoring kernel's epilogue: c_h = w_h * scale_q[h], four chains of
// c_h * ReLU(q_h . k) over the heads, their sum times the key's scale.
struct AppendedKey {
  int enabled;
  int fp4;               // keys in e2m1 (64 bytes per row) instead of e4m3
  const uint8_t *q;      // [B][H][128] e4m3 codes
  const float *q_scale;  // [B][H] or null (1)
  const void *w;         // [B][H]
  dsv4_dtype w_dt;
  const uint8_t *k_pages;
  const float *k_scales;
  const int32_t *block_table;
  int num_pages, max_blocks, H;
};

// Score of sequence b's appended entry j by the CTA's threads (thread t: head t / 16, dims
// 8 (t % 16) .. +7); -inf where the entry has no valid page. Every thread of the CTA calls it.
__device__ float appended_score(const AppendedKey &ap, int b, int64_t j, float *part /* [64] */) {
  const int tid = threadIdx.x, h = tid >> 4, sub = tid & 15;
  const int64_t lb = j / kPerPage;
  const int page = lb < ap.max_blocks ? ap.block_table[static_cast<size_t>(b) * ap.max_blocks + lb] : -1;
  const bool valid = page >= 0 && page < ap.num_pages;
  const size_t row = valid ? static_cast<size_t>(page) * kPerPage + static_cast<size_t>(j % kPerPage) : 0;
  float acc = 0.f;
  if (h < ap.H && valid) {
    const uint2 qq = *reinterpret_cast<const uint2 *>(ap.q + (static_cast<size_t>(b) * ap.H + h) * kRowBytes + 8 * sub);
    const uint32_t qw[2] = {qq.x, qq.y};
    float kv[8];
    if (ap.fp4) {  // dims 8 sub .. +7: one 32-bit word of 8 nibbles
      const uint32_t kw = *reinterpret_cast<const uint32_t *>(ap.k_pages + row * (kRowBytes / 2) + 4 * sub);
#pragma unroll
      for (int c = 0; c < 8; ++c) kv[c] = e2m1_to_float((kw >> (4 * c)) & 15u);
    } else {
      const uint2 kq = *reinterpret_cast<const uint2 *>(ap.k_pages + row * kRowBytes + 8 * sub);
      const uint32_t kw[2] = {kq.x, kq.y};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const float2 k0 = e4m3x2_to_float2(static_cast<uint16_t>(kw[u] & 0xFFFF));
        const float2 k1 = e4m3x2_to_float2(static_cast<uint16_t>(kw[u] >> 16));
        kv[4 * u] = k0.x;
        kv[4 * u + 1] = k0.y;
        kv[4 * u + 2] = k1.x;
        kv[4 * u + 3] = k1.y;
      }
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float2 q0 = e4m3x2_to_float2(static_cast<uint16_t>(qw[u] & 0xFFFF));
      const float2 q1 = e4m3x2_to_float2(static_cast<uint16_t>(qw[u] >> 16));
      acc = fmaf(q0.x, kv[4 * u], acc);
      acc = fmaf(q0.y, kv[4 * u + 1], acc);
      acc = fmaf(q1.x, kv[4 * u + 2], acc);
      acc = fmaf(q1.y, kv[4 * u + 3], acc);
    }
  }
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (sub == 0 && h < ap.H) part[h] = fmaxf(acc, 0.f);
  __syncthreads();
  float score = -INFINITY;
  if (tid == 0 && valid) {
    float c4[4] = {0.f, 0.f, 0.f, 0.f};
    for (int hh = 0; hh < ap.H; ++hh) {
      const float qs = ap.q_scale ? ap.q_scale[static_cast<size_t>(b) * ap.H + hh] : 1.0f;
      const float c = load_one_f(ap.w, ap.w_dt, static_cast<size_t>(b) * ap.H + hh) * qs;
      c4[hh & 3] = fmaf(c, part[hh], c4[hh & 3]);
    }
    const float sc = ap.k_scales[row];
    if (sc > 0.f) score = ((c4[0] + c4[1]) + (c4[2] + c4[3])) * sc;
  }
  return score;  // (thread 0's value)
}

template <int KPT, int NT>  // NT threads of KPT keys each: a CTA holds up to NT * KPT keys, all in registers
__global__ void __launch_bounds__(NT, 1) topk_scores_kernel(const float *scores, int64_t ld,
                                                                   const int32_t *n_entries, const int32_t *pos,
                                                                   int m, int64_t capacity, int slice,
                                                                   const TopkOut out, const AppendedKey ap,
                                                                   int release) {
  const int k = out.k;
  uint32_t *d_status = out.d_status;
  __shared__ float app_part[64];
  __shared__ float app_score;
  __shared__ int hist[2][256];  // this CTA's histogram of the current pass (double buffered)
  __shared__ int whist[NT / 32][256];  // first pass: one histogram per warp (no collisions between warps)
  __shared__ int ghist[256];    // the cluster's
  __shared__ int xch[2];        // read by the other CTAs: class members, kept keys
  __shared__ int warp_cnt[(NT / 32)], warp_base[(NT / 32)];
  __shared__ int sel_digit, sel_above, sel_count, bcast;
  const int b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_rank(), cs = cluster_size();
  const int64_t n = visible_entries(n_entries, pos, m, b, capacity, d_status, rank == 0 && tid == 0);
  const int64_t lo = static_cast<int64_t>(rank) * slice;
  const int cnt = static_cast<int>(n > lo ? (n - lo < slice ? n - lo : slice) : 0);
  pdl_wait();  // the scores come from the kernel before
  if (release) pdl_launch_dependents();  // only when a kernel of the same call follows
  // this step's appended entry, when it falls in this CTA's slice: scored here
  int app_i = -1;
  if (ap.enabled) {
    const int64_t p0 = pos[b], jn = (p0 + 1) / m - 1;
    if ((p0 + 1) % m == 0 && jn >= lo && jn < lo + cnt) app_i = static_cast<int>(jn - lo);
  }
  if (app_i >= 0) {  // uniform over the CTA
    const float sc = appended_score(ap, b, lo + app_i, app_part);
    if (tid == 0) app_score = sc;
    __syncthreads();
  }
  // warp w owns the contiguous run [w * 32 * KPT, (w + 1) * 32 * KPT) of the slice; its
  // lane l holds key r at position w * 32 * KPT + 32 r + l (coalesced loads, and the rounds
  // of the index-order walks below are the register index r)
  const int wbase = warp * 32 * KPT;
  const float *src = scores + static_cast<size_t>(b) * ld + lo;
  uint32_t key[KPT];
#pragma unroll
  for (int r = 0; r < KPT; ++r) {
    const int i = wbase + 32 * r + lane;
    float v = i < cnt ? __ldcs(src + i) : -INFINITY;
    if (i == app_i) v = app_score;
    key[r] = isfinite(v) ? float_order_key(v) : 0u;
  }
  uint32_t prefix = 0, mask = 0;
  int need = 0, total_valid = 0, kk = 0;
  bool whole_class = true;  // every key of the k-th key's class is kept (no ranks needed)
  auto pass = [&](int shift, int par) {  // the cluster histogram of digit `shift` of the matching keys
    if (shift == 24) {  // every key takes part: per-warp histograms, then summed
      for (int i = lane; i < 256; i += 32) whist[warp][i] = 0;
      __syncwarp();
#pragma unroll
      for (int r = 0; r < KPT; ++r)
        if (key[r] != 0u) atomicAdd(&whist[warp][key[r] >> 24], 1);
      __syncthreads();
      for (int i = tid; i < 256; i += NT) {
        int t = 0;
#pragma unroll 8
        for (int w = 0; w < NT / 32; ++w) t += whist[w][i];
        hist[par][i] = t;
      }
    } else {
      for (int i = tid; i < 256; i += NT) hist[par][i] = 0;
      __syncthreads();
#pragma unroll
      for (int r = 0; r < KPT; ++r)
        if (key[r] != 0u && (key[r] & mask) == prefix) atomicAdd(&hist[par][(key[r] >> shift) & 0xFF], 1);
    }
    cluster_sync_all();
    if (tid < 256) {  // all remote loads in flight before the first is used
      int v[kTkMaxCluster];
#pragma unroll
      for (int r = 0; r < kTkMaxCluster; ++r) v[r] = r < static_cast<int>(cs) ? ld_cluster(&hist[par][tid], r) : 0;
      int s = 0;
#pragma unroll
      for (int r = 0; r < kTkMaxCluster; ++r) s += v[r];
      ghist[tid] = s;
    }
    __syncthreads();
  };
  auto pick = [&](int want) {  // warp 0: the digit holding the want-th largest key
    if (tid < 32) {
      int c[8], tot = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) { c[u] = ghist[255 - tid * 8 - u]; tot += c[u]; }
      int incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (tid >= o) incl += v;
      }
      int run = incl - tot;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (run < want && run + c[u] >= want) {
          sel_digit = 255 - tid * 8 - u;
          sel_above = run;
          sel_count = c[u];
        }
        run += c[u];
      }
      const int all = __shfl_sync(0xFFFFFFFFu, incl, 31);
      if (tid == 0) bcast = all;
    }
    __syncthreads();
  };
  // The radix passes, each lambda called from one place (this code runs once per launch and
  // is fetched cold, so its length is its cost). The first pass also counts the valid keys
  // of the whole sequence (bcast): with fewer than k of them every valid key is kept;
  // otherwise its pick already found the digit of the k-th.
  bool partial = false;
  need = k;
#pragma unroll 1
  for (int shift = 24, par = 0;; shift -= 8, par ^= 1) {
    pass(shift, par);
    pick(need);
    if (shift == 24) {
      total_valid = bcast;
      kk = total_valid < k ? total_valid : k;
      partial = kk < total_valid;
      if (!partial) break;
    }
    prefix |= static_cast<uint32_t>(sel_digit) << shift;
    mask |= 0xFFu << shift;
    need -= sel_above;
    const int cntd = sel_count;
    __syncthreads();
    whole_class = cntd == need;
    if (whole_class || shift == 0) break;  // the whole class is taken, or the key is exact
  }
  auto above = [&](uint32_t kv) { return kv != 0u && (!partial || (kv & mask) > prefix); };
  auto in_class = [&](uint32_t kv) { return partial && kv != 0u && (kv & mask) == prefix; };
  // class members before this CTA and before each warp (only needed when the class is split)
  if (partial && !whole_class) {
    int e = 0;
#pragma unroll
    for (int r = 0; r < KPT; ++r) e += in_class(key[r]);
    e = warp_sum_int(e);
    if (lane == 0) warp_cnt[warp] = e;
    __syncthreads();
    if (tid == 0) {
      int run = 0;
      for (int w = 0; w < (NT / 32); ++w) { warp_base[w] = run; run += warp_cnt[w]; }
      xch[0] = run;
    }
    cluster_sync_all();
    if (warp == 0) {  // lane r reads CTA r
      int v = lane < static_cast<int>(rank) ? ld_cluster(&xch[0], lane) : 0;
      v = warp_sum_int(v);
      if (lane == 0) bcast = v;
    }
    __syncthreads();
  }
  const int eq_before = partial && !whole_class ? bcast + warp_base[warp] : 0;
  __syncthreads();
  // kept keys of each warp in index order (round r, then lane): counted, then written
  auto walk = [&](bool write, int at) {
    int e = eq_before, kept = 0;
#pragma unroll
    for (int r = 0; r < KPT; ++r) {
      const bool cl = in_class(key[r]);
      bool keep = above(key[r]) || (cl && whole_class);
      if (!whole_class) {  // uniform: the class is split, members are ranked in index order
        const unsigned clb = __ballot_sync(0xFFFFFFFFu, cl);
        keep = keep || (cl && e + __popc(clb & ((1u << lane) - 1u)) < need);
        e += __popc(clb);
      }
      const unsigned kb = __ballot_sync(0xFFFFFFFFu, keep);
      if (write && keep) {
        const int o = at + kept + __popc(kb & ((1u << lane) - 1u));
        if (o < k) out.put(b, o, static_cast<int32_t>(lo + wbase + 32 * r + lane), order_key_to_float(key[r]));
      }
      kept += __popc(kb);
    }
    return kept;
  };
  // the walk, from one place: counted (pass 0), then, with the counts of the warps before
  // and of the CTAs before exchanged, written (pass 1). When the whole class is kept (the
  // usual case) a warp's count needs no ranks: it is the number of its keys kept.
#pragma unroll 1
  for (int wp = 0, at = 0; wp < 2; ++wp) {
    int kept;
    if (wp == 0 && whole_class) {
      int c = 0;
#pragma unroll
      for (int r = 0; r < KPT; ++r) c += (above(key[r]) || in_class(key[r])) ? 1 : 0;
      kept = warp_sum_int(c);
    } else {
      kept = walk(wp == 1, at);
    }
    if (wp == 1) break;
    if (lane == 0) warp_cnt[warp] = kept;
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the warps' counts, lane w for warp w
      static_assert(NT / 32 <= 32, "one lane per warp");
      const int v = lane < NT / 32 ? warp_cnt[lane] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += u;
      }
      if (lane < NT / 32) warp_base[lane] = incl - v;
      if (lane == 31) xch[1] = incl;
    }
    cluster_sync_all();
    if (warp == 0) {  // lane r reads CTA r
      const int v = lane < static_cast<int>(cs) ? ld_cluster(&xch[1], lane) : 0;
      const int before = warp_sum_int(lane < static_cast<int>(rank) ? v : 0), all = warp_sum_int(v);
      if (lane == 0) {
        sel_above = before;
        sel_count = all;
      }
    }
    __syncthreads();
    at = sel_above + warp_base[warp];
  }
  if (rank == 0) {
    for (int i = sel_count + tid; i < k; i += NT) out.put(b, i, -1, -INFINITY);
  }
  cluster_sync_all();  // no CTA leaves while another may still read its shared memory
}

// ------------------------------------------------------------------------------------
// Per-sequence select: the k best keys of the candidate list, sorted (score desc,
// index asc), written as entry indices (+ scores); -1 / -inf padding.

__global__ void __launch_bounds__(kSelThreads) topk_select_kernel(const unsigned long long *cand, int64_t stride,
                                                                  const int *cand_count, int k, int32_t *idx,
                                                                  float *scores, uint32_t *d_status, int smem_keys,
                                                                  int release) {
  pdl_wait();
  if (release) pdl_launch_dependents();  // only when a kernel of the same call follows
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

// Rows of 128 values: e4m3 (128 bytes each), or e2m1 (fp4: 64 packed bytes each, landing in
// shared memory as 128-byte rows with each 8 bytes of values followed by 8 bytes of gap, the
// operand layout of the f8f6f4 MMA's e2m1 type). 128B swizzle either way.
bool make_rows_map(CUtensorMap *map, const void *base, uint64_t rows, uint32_t box_rows, bool fp4 = false) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kRowBytes), static_cast<cuuint64_t>(rows)};  // values
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(fp4 ? kRowBytes / 2 : kRowBytes)};          // bytes
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kRowBytes), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, fp4 ? CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
            const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

int tc_grid() { return sm_count(); }

int64_t capacity_of(const IndexerLaunch &p) {
  return static_cast<int64_t>(p.max_blocks) * (DSV4_PAGE_POSITIONS / p.m);
}
int64_t score_ld(const IndexerLaunch &p) { return (capacity_of(p) + 3) / 4 * 4; }

// CTAs per sequence of the top-k cluster: enough for a slice to fit in shared memory, and
// as many as keep the batch within one wave of SMs (a power of two, at most 16)
// CTAs per sequence of the top-k: one while the sequence's entries fit in one CTA's
// registers (no cluster barriers at all), else the smallest power-of-two cluster that fits
int tk_cluster(const IndexerLaunch &p) {
  if (capacity_of(p) <= kTkSolo) return 1;
  int need = 1;
  while (static_cast<int64_t>(need) * kTkSlice < capacity_of(p)) need <<= 1;
  while (need < 8 && static_cast<int64_t>(need) * 2 * p.B <= sm_count()) need <<= 1;  // more CTAs while they fit one wave
  return need;
}
int tk_slice(const IndexerLaunch &p) {
  const int cs = tk_cluster(p);
  return static_cast<int>((capacity_of(p) + cs - 1) / cs);
}

// candidate list length per sequence (CUDA-core path: every entry)
int64_t cand_stride(const IndexerLaunch &p) {
  if (indexer_uses_tensor_cores(p)) return 0;
  const int64_t capacity = capacity_of(p);
  return capacity > 0 ? capacity : 1;
}

// shared memory of the scoring kernel: TcSmem plus the tile prefix and visible counts
size_t tc_tail_bytes(int B) { return 1024 + (2 * static_cast<size_t>(B) + 1) * 8; }

template <int H>
int tc_stages(int B) {
  return sizeof(TcSmem<H, kStagesHi>) + tc_tail_bytes(B) <= 227 * 1024 ? kStagesHi : kStagesLo;
}

template <int H>
cudaError_t launch_tc(const IndexerLaunch &p, float *scores, cudaStream_t st, int64_t ld = 0) {
  TcParams tp{};
  const bool fp4 = p.k_dt == DSV4_FP4E2M1;
  if (!make_rows_map(&tp.tmap_k, p.k_pages, static_cast<uint64_t>(p.num_pages) * kPerPage, kPerPage, fp4))
    return cudaErrorInvalidValue;
  tp.keys_fp4 = fp4 ? 1 : 0;
  if (!make_rows_map(&tp.tmap_q, p.q, static_cast<uint64_t>(p.B) * H, H)) return cudaErrorInvalidValue;
  tp.k_scales = p.k_scales;
  tp.block_table = p.block_table;
  tp.num_pages = p.num_pages;
  tp.max_blocks = p.max_blocks;
  tp.q_scale = p.q_scale;
  tp.w = p.w;
  tp.w_dt = p.w_dt;
  tp.B = p.B;
  tp.m = p.m;
  tp.n_entries = p.n_entries;
  tp.pos = p.pos;
  tp.scores = scores;
  tp.ld = ld > 0 ? ld : score_ld(p);
  tp.d_status = p.d_status;
  tp.before_append = p.before_append ? 1 : 0;
  tp.release = p.idx != nullptr || p.release_next ? 1 : 0;  // the top-k kernel, or a kernel of the call, follows
  // six stages in flight where shared memory allows, else five
  const size_t tail = tc_tail_bytes(p.B);
  if (tc_stages<H>(p.B) == kStagesHi) {
    const size_t smem = sizeof(TcSmem<H, kStagesHi>) + tail;
    cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<H, kStagesHi>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(indexer_tc_kernel<H, kStagesHi>, dim3(tc_grid()), dim3(kIxThreads), smem, st, 1, tp);
  }
  const size_t smem = sizeof(TcSmem<H, kStagesLo>) + tail;
  cudaError_t e = cudaFuncSetAttribute(indexer_tc_kernel<H, kStagesLo>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(indexer_tc_kernel<H, kStagesLo>, dim3(tc_grid()), dim3(kIxThreads), smem, st, 1, tp);
}

}  // namespace

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

bool indexer_uses_tensor_cores(const IndexerLaunch &p) {
  const bool keys_ok = p.k_dt == DSV4_FP8E4M3 ||
                       (p.k_dt == DSV4_FP4E2M1 && (reinterpret_cast<uintptr_t>(p.k_pages) & 31u) == 0);
  return keys_ok && p.q_dt == DSV4_FP8E4M3 && p.Dq == kRowBytes &&
         (p.H == 32 || p.H == 64) && p.m == 4 && p.k >= 1 && p.k <= 2048 && p.q_rope_dims == 0 &&
         p.B <= 512 && static_cast<int64_t>(p.max_blocks) * (DSV4_PAGE_POSITIONS / p.m) <= kTkMaxCluster * kTkSlice;
}

size_t indexer_workspace_bytes(const IndexerLaunch &p) {
  size_t bytes = align_up(static_cast<size_t>(p.B) * sizeof(int), 256) +
                 align_up(static_cast<size_t>(p.B) * cand_stride(p) * sizeof(unsigned long long), 256);
  if (indexer_uses_tensor_cores(p)) bytes += align_up(static_cast<size_t>(p.B) * score_ld(p) * sizeof(float), 256);
  return bytes;
}


cudaError_t launch_indexer_topk(const IndexerLaunch &p0, void *ws, cudaStream_t st) {
  return launch_indexer_part(p0, ws, st, 0);
}

int64_t indexer_score_capacity(const IndexerLaunch &p) { return capacity_of(p); }

cudaError_t launch_indexer_scores(const IndexerLaunch &p, float *scores, int64_t ld, cudaStream_t st) {
  IndexerLaunch q = p;
  q.release_next = false;
  return q.H == 32 ? launch_tc<32>(q, scores, st, ld) : launch_tc<64>(q, scores, st, ld);
}

cudaError_t launch_indexer_part(const IndexerLaunch &p0, void *ws, cudaStream_t st, int part) {
  IndexerLaunch p = p0;
  p.rope_theta1 = rope_theta1(p.rope_base, p.q_rope_dims);
  char *w = static_cast<char *>(ws);
  int *cand_count = reinterpret_cast<int *>(w);
  w += align_up(static_cast<size_t>(p.B) * sizeof(int), 256);
  unsigned long long *cand = reinterpret_cast<unsigned long long *>(w);
  const int64_t stride = cand_stride(p);
  w += align_up(static_cast<size_t>(p.B) * stride * sizeof(unsigned long long), 256);
  cudaError_t e = cudaSuccess;
  if (indexer_uses_tensor_cores(p)) {
    float *scores = reinterpret_cast<float *>(w);
    if (part != 2) {
      e = p.H == 32 ? launch_tc<32>(p, scores, st) : launch_tc<64>(p, scores, st);
      if (e != cudaSuccess || part == 1) return e;
    }
    AppendedKey ap{};
    if (p.before_append && !p.n_entries) {
      ap.enabled = 1;
      ap.fp4 = p.k_dt == DSV4_FP4E2M1 ? 1 : 0;
      ap.q = static_cast<const uint8_t *>(p.q);
      ap.q_scale = p.q_scale;
      ap.w = p.w;
      ap.w_dt = p.w_dt;
      ap.k_pages = static_cast<const uint8_t *>(p.k_pages);
      ap.k_scales = p.k_scales;
      ap.block_table = p.block_table;
      ap.num_pages = p.num_pages;
      ap.max_blocks = p.max_blocks;
      ap.H = p.H;
    }
    TopkOut out{};
    out.idx = p.idx;
    out.scores = p.scores;
    out.k = p.k;
    out.d_status = p.d_status;
    const int rel = p.release_next ? 1 : 0;
    const int cs = tk_cluster(p), slice = tk_slice(p);
    auto launch_k = [&](auto kern, int nt) -> cudaError_t {
      if (cs > 8) {
        const cudaError_t a = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (a != cudaSuccess) return a;
      }
      return launch_pdl(kern, dim3(static_cast<unsigned>(cs), static_cast<unsigned>(p.B)), dim3(nt), 0, st, cs,
                        static_cast<const float *>(scores), score_ld(p), p.n_entries, p.pos, p.m, capacity_of(p),
                        slice, out, ap, rel);
    };
    if (slice <= 8 * kTkThreads) return launch_k(topk_scores_kernel<8, kTkThreads>, kTkThreads);
    if (slice <= 16 * kTkThreads) return launch_k(topk_scores_kernel<16, kTkThreads>, kTkThreads);
    return launch_k(topk_scores_kernel<24, kTkThreads>, kTkThreads);
  } else {
    e = cudaMemsetAsync(cand_count, 0, static_cast<size_t>(p.B) * sizeof(int), st);
    if (e != cudaSuccess) return e;
    const int64_t capacity = capacity_of(p);
    dim3 grid(static_cast<unsigned>((capacity + 255) / 256), p.B);
    const size_t smem = (static_cast<size_t>(p.H) * p.Dq + p.H) * sizeof(float);
    e = cudaFuncSetAttribute(indexer_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(indexer_simt_kernel, grid, dim3(256), smem, st, 1, p, cand, stride, cand_count);
    if (e != cudaSuccess) return e;
  }
  // merge candidate lists: stage up to ~200 KB of candidates in shared memory
  const int smem_keys = static_cast<int>(std::min<int64_t>(stride + kMaxSortK, 25600));
  const size_t ssmem = static_cast<size_t>(smem_keys) * sizeof(unsigned long long);
  e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)ssmem);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_select_kernel, dim3(p.B), dim3(kSelThreads), ssmem, st, 1,
                    static_cast<const unsigned long long *>(cand), stride, static_cast<const int *>(cand_count), p.k,
                    p.idx, p.scores, p.d_status, smem_keys, p.release_next ? 1 : 0);
}

}  // namespace dsv4
