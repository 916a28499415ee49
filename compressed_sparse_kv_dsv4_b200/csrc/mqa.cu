// Shared-K/V multi-query attention of one decode query per sequence, with the query
// rotated by RoPE_pos and the output rotated back by -pos (steps (3) and (4) of the decode
// method; vLLM "four moves": shared K/V + inverse RoPE, sparse attention over compressed
// tokens united with a short sliding window; SGLang "Shadow radix": SWA-128 + C4 top-512
// or C128 dense).
//
// Keys of sequence s (V = K): window positions max(0,p-W+1)..p, then the selected entries
// idx[s][0..k) (C4) or all visible entries (C128).
//
// Tensor-core path (bf16/fp8 caches, D = 512, H = 64):
//   mqa_query_kernel: the query rotated by RoPE_pos once per sequence, as fp16 scaled per
//     head by a power of two (fp8 caches) or bf16;
//   mqa_tc_kernel: one thread-block cluster of cs CTAs per sequence, CTA r on a contiguous
//     run of the sequence's 64-key chunks, with warp roles connected by mbarriers:
//       metadata warp: row address + scale of every key (idx -> block table -> scale);
//       gather warps:  64 rows into a 128B-swizzled K-major tile (fp8 -> fp16 exact, the
//                      row scale folded in; bf16 copied), and the prepared query;
//       MMA warp:      S[64 heads x 64 keys] = Q K^T (tcgen05 kind::f16, M = 64, TMEM lanes
//                      16..31), then O[64 x 512] += P K (the same tile read MN-major, lanes 0..15);
//       softmax warps: online softmax in log2 units with a lazy reference max, P to smem.
//     The MMA warp issues S of chunk n + 1 (two S buffers in TMEM) while the softmax warps
//     work on chunk n. At the end the cluster merges its partials: (max, sum) exchanged
//     per head and each CTA's O staged per owner in its freed tile buffers, both passed
//     through global memory (L2 moves them several times faster than the cluster's
//     shared-memory network); CTA r weighs and sums its slabs, normalizes, inverse-rotates
//     and stores columns [r * 512/cs, (r+1) * 512/cs).
// CUDA-core path (any dtype, D <= 1024): mqa_simt_kernel, one CTA per (head, sequence).
#include "common.cuh"
#include "internal.h"

namespace dsv4 {

namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// ------------------------------------------------------------------------------------
// per-sequence key list

struct KeyList {
  int64_t pos, nw, nsel, n_entries;
};

__device__ __forceinline__ KeyList key_list(const MqaLaunch &p, int b, bool report_it) {
  KeyList L;
  L.pos = p.pos[b];
  const int64_t capacity = static_cast<int64_t>(p.max_blocks) * (DSV4_PAGE_POSITIONS / p.m);
  int64_t n = p.n_entries ? static_cast<int64_t>(p.n_entries[b]) : (L.pos + 1) / p.m;
  if (n < 0) n = 0;
  if (n > capacity) {
    if (report_it) report(p.d_status, DSV4_DEV_BAD_LENGTH);
    n = capacity;
  }
  L.n_entries = n;
  if (L.pos < 0) {
    if (report_it) report(p.d_status, DSV4_DEV_BAD_LENGTH);
    L.nw = 0; L.nsel = 0;
    return L;
  }
  L.nw = L.pos + 1 < p.W ? L.pos + 1 : p.W;
  L.nsel = p.idx ? p.k : n;
  return L;
}

// address and scale of key t of a sequence's list; nullptr = skipped (no contribution)
__device__ __forceinline__ const uint8_t *key_row(const MqaLaunch &p, int b, const KeyList &L, int64_t t,
                                                  float *scale) {
  const size_t esz = dtype_size(p.kv_dt);
  *scale = 1.0f;
  if (t < L.nw) {
    const int64_t pw = L.pos - L.nw + 1 + t;
    const size_t slot = static_cast<size_t>(b) * p.W + static_cast<size_t>(pw % p.W);
    if (p.kv_dt == DSV4_FP8E4M3) *scale = p.ring_scales[slot];
    return static_cast<const uint8_t *>(p.ring_rows) + slot * p.D * esz;
  }
  const int64_t u = t - L.nw;
  if (u >= L.nsel) return nullptr;
  int64_t j = u;
  if (p.idx) {
    j = p.idx[static_cast<size_t>(b) * p.k + u];
    if (j < 0) return nullptr;  // padding
    if (j >= L.n_entries) {
      report(p.d_status, DSV4_DEV_BAD_INDEX);
      return nullptr;
    }
  }
  const int per_page = DSV4_PAGE_POSITIONS / p.m;
  const int page = p.block_table[static_cast<size_t>(b) * p.max_blocks + j / per_page];
  if (page < 0 || page >= p.num_pages) {
    report(p.d_status, DSV4_DEV_BAD_PAGE);
    return nullptr;
  }
  const size_t row = static_cast<size_t>(page) * per_page + static_cast<size_t>(j % per_page);
  if (p.kv_dt == DSV4_FP8E4M3) *scale = p.scales[row];
  return static_cast<const uint8_t *>(p.pages) + row * p.D * esz;
}

// ------------------------------------------------------------------------------------
// tensor-core kernel: one thread-block cluster of cs CTAs per sequence; CTA r takes a
// contiguous run of the sequence's 64-key chunks, and the cluster merges the CTAs' partial
// results through L2 (the workspace) at the end.

constexpr int kH = 64, kD = 512, kCh = 64;
constexpr int kAtom = kCh * 128;  // one 64-dim column block of a 64-row tile: 8 KB
constexpr int kMetaSlots = 4;     // chunks whose key metadata is resolved ahead
// roles: warps 0-3 softmax + output (TMEM lane quadrant = warp), warps 4-7 gather, warp 8
// MMA issue (and TMEM allocation), warp 9 key metadata
constexpr int kSoftWarp0 = 0, kGatherWarp0 = 4, kMmaWarp = 8, kMetaWarp = 9;
constexpr int kThreads = 320;
constexpr int kMaxCluster = 16;

struct alignas(1024) MqaSmem {
  uint8_t q[kD / 64][kH * 128];  // 64 KB, K-major SW128, 8 atoms of 64 dims
  union {
    uint8_t k[2][kD / 64][kCh * 128];  // 2 x 64 KB key tiles (stage = chunk parity)
    float rbuf[kH * kD];               // after the last MMA: this CTA's weighted O, one slab per owner
  };
  uint8_t p[kH * 128];                   // 8 KB: P[64 heads][64 keys], K-major SW128
  const uint8_t *mrow[kMetaSlots][kCh];  // row address of each key of a chunk (nullptr: none)
  float mscale[kMetaSlots][kCh];         // its row scale
  float rscale[2][kCh];                  // row scale per key of a staged tile (0: no key)
  int ec[2];                             // tile exponent: K rows hold code * scale * 2^-ec
  float qinv[kH];                        // 2^-e of the per-head query scale
  float red_m[kH], red_l[kH];            // this CTA's reference max and sum per head (read by the cluster)
  float inv_l[kH], lse[kH];              // 1 / the cluster's total sum, log-sum-exp, per head
  float wsrc[kMaxCluster][kH];           // weight 2^(R - M) of each cluster CTA's partial, per head
  uint64_t meta_full[kMetaSlots], meta_empty[kMetaSlots];
  uint64_t k_full[2], k_empty[2], q_full, s_full[2], s_empty[2], p_full, o_full, mma_done, part_full;
  uint32_t tmem_base;
  int abort_flag;
  int dry[kThreads / 32];  // per warp: 1 during its first, dry pass (see the kernel)
};

static_assert(sizeof(MqaSmem) + 1024 <= 227 * 1024, "attention shared memory exceeds one SM");

struct MqaTcParams {
  MqaLaunch a;
  float scale_log2;
  uint16_t *qp;    // [B][H][D] query rotated by RoPE_pos, fp16 (scaled per head) or bf16
  float *qinv;     // [B][H] 2^-e undoing the per-head scale (1 for bf16)
  float *part;     // [B][cs][cs - 1] slabs [H][D / cs]: CTA src's O for owner dst != src
  float *red;      // [B][cs][2][H]: each CTA's reference max R and sum l per head
};

// The dry pass of this warp: read from shared memory at every use, so that the compiler
// keeps one copy of the code for both passes.
__device__ __forceinline__ bool dry_pass(const MqaSmem &S) {
  return *reinterpret_cast<const volatile int *>(&S.dry[threadIdx.x >> 5]) != 0;
}

// Operands of the two MMAs. fp8 caches: fp16 (e4m3 -> fp16 is exact, and fp16 keeps 11
// significand bits of the rotated query and of P); bf16 caches: bf16.
__device__ __forceinline__ bool fp16_operands(const MqaLaunch &p) { return p.kv_dt == DSV4_FP8E4M3; }

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

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
// every thread of every CTA of the cluster; orders the memory writes before it with the reads after it
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 16-byte run c of row h of a merge slab: runs are XOR-swizzled by h so that the 16 rows a warp
// writes at once land in different banks
__device__ __forceinline__ int slab_run(int h, int c) { return c ^ (h & 7); }

// This CTA's chunks of its sequence: [lo, hi) of the sequence's C chunks.
struct ChunkRange {
  int b;
  long long lo, hi;
};

// ---- warp 9: row address and scale of every key of up to kMetaSlots chunks at a time.
// The idx -> block table -> scale chain is staged over all keys of the batch, so its three
// memory latencies are paid once per batch.
__device__ void meta_role(const MqaLaunch &p, MqaSmem &S, const KeyList &L, const ChunkRange &cr) {
  const int lane = threadIdx.x & 31, b = cr.b;
  // 32-bit arithmetic throughout (this code runs once per launch, so its length is its cost):
  // entries per page (m and the page size are powers of two), the window's first ring slot
  const int per_shift = __ffs(DSV4_PAGE_POSITIONS) - __ffs(p.m), per_mask = (1 << per_shift) - 1;
  const int nw = static_cast<int>(L.nw), W = p.W;
  const int w0 = nw > 0 ? static_cast<int>((L.pos - L.nw + 1) % p.W) : 0;
  const size_t row_bytes = static_cast<size_t>(p.D) * dtype_size(p.kv_dt);
  const bool fp8 = p.kv_dt == DSV4_FP8E4M3;
  const int32_t *idx_b = p.idx ? p.idx + static_cast<size_t>(b) * p.k : nullptr;
  const int32_t *bt_b = p.block_table + static_cast<size_t>(b) * p.max_blocks;
  const uint8_t *ring_b = static_cast<const uint8_t *>(p.ring_rows) + static_cast<size_t>(b) * W * row_bytes;
  const float *ring_sc_b = fp8 ? p.ring_scales + static_cast<size_t>(b) * W : nullptr;
  constexpr int kKeys = kMetaSlots * 2;  // keys per lane per batch
  for (long long g0 = cr.lo; g0 < cr.hi; g0 += kMetaSlots) {
    const int nb = static_cast<int>(cr.hi - g0 < kMetaSlots ? cr.hi - g0 : kMetaSlots);
    bool ok = true;
    for (int i = 0; i < nb; ++i) {
      const long long n = g0 + i - cr.lo;
      if (n >= kMetaSlots && lane == 0 &&
          !mbar_wait(&S.meta_empty[n % kMetaSlots], static_cast<uint32_t>((n / kMetaSlots - 1) & 1), &S.abort_flag))
        ok = false;
    }
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      return;
    }
    // Three stages, each with the loads of all kKeys keys issued together: every load reads
    // a clamped, always-valid address and the result is selected afterwards, so no branch
    // separates them; bad indices and pages are reported after the loads, so no atomic sits
    // between two loads. kind: 0 none, 1 window row, 2 selected entry.
    int kind[kKeys], t[kKeys], j[kKeys];
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {
      const int i = u >> 1;
      t[u] = static_cast<int>(g0 + i) * kCh + lane + 32 * (u & 1);
      kind[u] = i >= nb ? 0 : (t[u] < nw ? 1 : (t[u] - nw < L.nsel ? 2 : 0));
    }
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {  // stage 1: list position -> entry index (idx load)
      j[u] = kind[u] == 2 ? t[u] - nw : 0;
      if (idx_b) j[u] = idx_b[j[u]];
    }
    bool bad_index = false, bad_page = false;
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {  // entries out of range and padding: no key
      if (kind[u] == 2 && j[u] >= L.n_entries) bad_index = true;
      if (kind[u] == 2 && (j[u] < 0 || j[u] >= L.n_entries)) kind[u] = 0;
    }
    int page[kKeys];
#pragma unroll
    for (int u = 0; u < kKeys; ++u)  // stage 2: entry -> physical page (block table load)
      page[u] = bt_b[kind[u] == 2 ? j[u] >> per_shift : 0];
    size_t row[kKeys];  // window: ring slot of the sequence; entry: row of the page pool
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {
      row[u] = 0;
      if (kind[u] == 1) {
        int slot = w0 + t[u];  // t < nw <= W
        if (slot >= W) slot -= W;
        row[u] = static_cast<size_t>(slot);
      } else if (kind[u] == 2) {
        if (page[u] < 0 || page[u] >= p.num_pages) {
          bad_page = true;
          kind[u] = 0;
        } else {
          row[u] = (static_cast<size_t>(page[u]) << per_shift) | static_cast<size_t>(j[u] & per_mask);
        }
      }
    }
    float sc[kKeys];
#pragma unroll
    for (int u = 0; u < kKeys; ++u)  // stage 3: row scale
      sc[u] = fp8 ? (kind[u] == 1 ? ring_sc_b : p.scales)[row[u]] : 1.0f;
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {
      const int i = u >> 1;
      const uint8_t *rp = kind[u] == 0 ? nullptr
                                       : (kind[u] == 1 ? ring_b : static_cast<const uint8_t *>(p.pages)) +
                                             row[u] * row_bytes;
      if (i < nb) {
        const int slot = static_cast<int>((g0 + i - cr.lo) % kMetaSlots);
        S.mrow[slot][lane + 32 * (u & 1)] = rp;
        S.mscale[slot][lane + 32 * (u & 1)] = rp ? sc[u] : 0.f;
        // the gather of this CTA's third and later chunks waits for a free tile stage: their
        // rows travel to L2 meanwhile
        if (rp && g0 + i - cr.lo >= 2) bulk_prefetch_l2(rp, static_cast<uint32_t>(row_bytes));
      }
    }
    if (bad_index) report(p.d_status, DSV4_DEV_BAD_INDEX);
    if (bad_page) report(p.d_status, DSV4_DEV_BAD_PAGE);
    __syncwarp();
    if (lane == 0)
      for (int i = 0; i < nb; ++i) mbar_arrive(&S.meta_full[(g0 + i - cr.lo) % kMetaSlots]);
  }
}

// ---- the query of every sequence, rotated by RoPE_pos once: bf16, or fp16 scaled per
// head by a power of two (qinv undoes it in the logits) so that |q| < 2^14 whatever the
// input range. grid (B, H / 8), 128 threads (small enough to share an SM with the indexer):
// thread t owns dims 32 (t & 15) .. +31 of head 8 blockIdx.y + t / 16. It reads only the
// caller's query and writes only qp/qinv, which no kernel before it in the same call reads,
// so it releases the next kernel at once and runs before its own pdl_wait().
__global__ void __launch_bounds__(128) mqa_query_kernel(const MqaTcParams P) {
  pdl_launch_dependents();
  const MqaLaunch &p = P.a;
  __shared__ float cs[kD / 2], sn[kD / 2];
  const int b = blockIdx.x, t = threadIdx.x, h = blockIdx.y * 8 + (t >> 4), d0 = (t & 15) * 32;
  const bool f16 = fp16_operands(p);
  const int half = p.rope_dims / 2, rope0 = kD - p.rope_dims;
  const int64_t pos = p.pos[b];
  for (int i = t; i < half; i += 128) rope_cos_sin(pos, i, p.rope_theta1, &cs[i], &sn[i]);
  const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.q) +
                                                     (static_cast<size_t>(b) * kH + h) * kD + d0);
  uint4 raw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) raw[i] = __ldg(src + i);
  __syncthreads();
  float x[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x[i][2 * u] = __uint_as_float(v[u] << 16);
      x[i][2 * u + 1] = __uint_as_float(v[u] & 0xFFFF0000u);
    }
  }
  if (p.q_norm_gamma) {  // RMSNorm of the head (its 16 threads are consecutive lanes), times gamma
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 8; ++u) ss += x[i][u] * x[i][u];
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
    const float rs = 1.0f / sqrtf(ss / static_cast<float>(kD) + p.q_norm_eps);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 8; ++u) x[i][u] = x[i][u] * rs * __ldg(p.q_norm_gamma + d0 + i * 8 + u);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {  // the 8 values of run i, rotated where they are rope dims
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int d = d0 + i * 8 + 2 * u;
      if (d >= rope0) {
        const float c = cs[(d - rope0) >> 1], sv = sn[(d - rope0) >> 1];
        const float x0 = x[i][2 * u], x1 = x[i][2 * u + 1];
        x[i][2 * u] = x0 * c - x1 * sv;
        x[i][2 * u + 1] = x0 * sv + x1 * c;
      }
    }
  }
  float qs = 1.0f, qi = 1.0f;
  if (f16) {
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int u = 0; u < 8; ++u) am = fmaxf(am, fabsf(x[i][u]));
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
    int e = 0;
    if (am > 0.f) frexpf(am, &e);  // am < 2^e
    qi = am > 0.f ? ldexpf(1.0f, e - 14) : 1.0f;
    qs = am > 0.f ? ldexpf(1.0f, 14 - e) : 1.0f;
  }
  uint4 *dst = reinterpret_cast<uint4 *>(P.qp + (static_cast<size_t>(b) * kH + h) * kD + d0);
#pragma unroll
  for (int i = 0; i < 4; ++i)
    dst[i] = f16 ? make_uint4(pack_f16x2(x[i][0] * qs, x[i][1] * qs), pack_f16x2(x[i][2] * qs, x[i][3] * qs),
                              pack_f16x2(x[i][4] * qs, x[i][5] * qs), pack_f16x2(x[i][6] * qs, x[i][7] * qs))
                 : make_uint4(pack_bf16x2(x[i][0], x[i][1]), pack_bf16x2(x[i][2], x[i][3]),
                              pack_bf16x2(x[i][4], x[i][5]), pack_bf16x2(x[i][6], x[i][7]));
  if ((t & 15) == 0) P.qinv[static_cast<size_t>(b) * kH + h] = qi;
  pdl_wait();  // completes only after the kernel before it: the chain of waits stays unbroken
}

// ---- warps 4-7 (gw = 0..3): query of a new segment and the key tiles. Query: warp gw
// copies the prepared rows of heads 16gw .. 16gw+15 into their swizzled homes (lane l owns
// 16-byte runs l and l + 32 of each) and their scales.
__device__ __forceinline__ void query_issue(const MqaTcParams &P, MqaSmem &S, int b, int gw, int lane) {
  const uint16_t *q = P.qp + static_cast<size_t>(b) * kH * kD;
#pragma unroll 4
  for (int hh = 0; hh < 16; ++hh) {
    const int h = gw * 16 + hh;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int seg = lane + 32 * r;
      cp_async16(&S.q[seg >> 3][0] + sw128_offset(h, seg & 7), q + (static_cast<size_t>(h) * kD + seg * 8));
    }
  }
  cp_async_commit();
}

__device__ __forceinline__ void query_finish(const MqaTcParams &P, MqaSmem &S, int b, int gw, int lane) {
  if (lane < 16) S.qinv[gw * 16 + lane] = P.qinv[static_cast<size_t>(b) * kH + gw * 16 + lane];
  cp_async_wait_all();
}

// Key tile of one chunk: warp gw fills rows 16gw .. 16gw+15. fp8 rows (32 runs of 16
// codes): lane l loads run l of each row and stores it as fp16 code * (scale * 2^-ec), ec
// the exponent of the chunk's largest row scale, so every tile value stays within +-448.
// bf16 rows (64 runs of 8 values) are copied as they are.
__device__ __forceinline__ void gather_issue_bf16(const MqaSmem &S, uint8_t *kt, int ms, int gw, int lane) {
#pragma unroll 4
  for (int rr = 0; rr < 16; ++rr) {
    const int row = gw * 16 + rr;
    const uint8_t *rp = S.mrow[ms][row];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int seg = lane + 32 * r;
      uint8_t *dst = kt + (seg >> 3) * kAtom + sw128_offset(row, seg & 7);
      if (rp) cp_async16(dst, rp + seg * 16);
      else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
  cp_async_commit();
}

__device__ __forceinline__ void gather_load_fp8(const MqaSmem &S, int ms, int gw, int lane, uint4 (&v)[16],
                                                bool none) {
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const uint8_t *rp = none ? nullptr : S.mrow[ms][gw * 16 + rr];
    v[rr] = rp ? __ldg(reinterpret_cast<const uint4 *>(rp + lane * 16)) : make_uint4(0, 0, 0, 0);
  }
}

// 2^e as a float (exact; e outside the normal range goes through ldexpf)
__device__ __forceinline__ float pow2f(int e) {
  return (e >= -126 && e <= 127) ? __int_as_float((127 + e) << 23) : ldexpf(1.0f, e);
}

// Converts and stores the rows in v (chunk of metadata slot ms); with next >= 0, each row's
// registers are refilled at once with the same row of the chunk in slot next, so those loads
// are in flight while the rest converts.
__device__ __forceinline__ void gather_store_fp8(MqaSmem &S, uint8_t *kt, int ms, int ec, int gw, int lane, uint4 (&v)[16],
                                                 int next) {
  const int atom = lane >> 2, c0 = (lane & 3) * 2;
  const float f = pow2f(-ec);  // row scale * 2^-ec: exact (a power-of-two factor)
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const int row = gw * 16 + rr;
    const __half2 sc2 = __float2half2_rn(S.mscale[ms][row] * f);
    const uint32_t w[4] = {v[rr].x, v[rr].y, v[rr].z, v[rr].w};
    uint32_t o[8];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[u] & 0xFFFF), __NV_E4M3);
      __half2_raw cc = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[u] >> 16), __NV_E4M3);
      __half2 ha = __hmul2(*reinterpret_cast<__half2 *>(&a), sc2);
      __half2 hc = __hmul2(*reinterpret_cast<__half2 *>(&cc), sc2);
      o[2 * u] = *reinterpret_cast<uint32_t *>(&ha);
      o[2 * u + 1] = *reinterpret_cast<uint32_t *>(&hc);
    }
    uint8_t *base = kt + atom * kAtom;
    *reinterpret_cast<uint4 *>(base + sw128_offset(row, c0)) = make_uint4(o[0], o[1], o[2], o[3]);
    *reinterpret_cast<uint4 *>(base + sw128_offset(row, c0 + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
    if (next >= 0) {
      const uint8_t *rp = S.mrow[next][row];
      v[rr] = rp ? __ldg(reinterpret_cast<const uint4 *>(rp + lane * 16)) : make_uint4(0, 0, 0, 0);
    }
  }
}

// fp8 rows are software-pipelined: while chunk n is converted, the registers of each row are
// refilled with the same row of chunk n + 1, so the memory latency of chunk n + 1 overlaps the
// conversion and the wait for its tile stage. The metadata of chunk n + 1 is awaited in
// iteration n: early, or, when chunk n + 1 opens a new metadata batch (which the metadata
// warp resolves only once every slot of the batch before is released, this chunk's
// included), after chunk n released its slot (and its rows are loaded then).
__device__ void gather_role(const MqaTcParams &P, MqaSmem &S, const ChunkRange &cr) {
  const MqaLaunch &p = P.a;
  const int lane = threadIdx.x & 31, gw = (threadIdx.x >> 5) - kGatherWarp0;
  const bool fp8 = p.kv_dt == DSV4_FP8E4M3;
  // the dry pass goes once through the loop with no wait, no arrival and no row read
  const bool dry = dry_pass(S);
  const long long nc = dry ? (cr.lo < cr.hi ? 1 : 0) : cr.hi - cr.lo;
  if (nc > 0 && !dry) query_issue(P, S, cr.b, gw, lane);
  uint4 v[16];  // rows of the chunk at hand (fp8)
  if (nc > 0) {
    const bool ok = dry || mbar_wait(&S.meta_full[0], 0u, &S.abort_flag);
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      return;
    }
    if (fp8) gather_load_fp8(S, 0, gw, lane, v, dry);
  }
  for (long long n = 0; n < nc; ++n) {
    const int s = static_cast<int>(n & 1), ms = static_cast<int>(n % kMetaSlots);
    bool ok = true;
    const bool ahead = n + 1 < nc && (n + 1) % kMetaSlots != 0;
    if (ahead)
      ok = mbar_wait(&S.meta_full[(n + 1) % kMetaSlots], static_cast<uint32_t>(((n + 1) / kMetaSlots) & 1),
                     &S.abort_flag);
    if (ok && n >= 2) ok = mbar_wait(&S.k_empty[s], static_cast<uint32_t>((n / 2 - 1) & 1), &S.abort_flag);
    // (the dry pass reads placeholder metadata below and converts zero rows)
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      break;
    }
    // the query copy (first chunk) and the key rows are in flight together; the tile is
    // finished first, then the query
    uint8_t *kt = &S.k[s][0][0];
    // chunk exponent (every warp derives the same one) and the scales softmax reads
    const float smax = warp_max(fmaxf(S.mscale[ms][lane], S.mscale[ms][lane + 32]));
    int ec = 0;
    if (fp8) frexpf(smax, &ec);  // largest scale = f * 2^ec, f in [0.5, 1)
    if (lane < 16) S.rscale[s][gw * 16 + lane] = S.mscale[ms][gw * 16 + lane];
    if (gw == 0 && lane == 0 && !dry) S.ec[s] = ec;
    if (fp8) {
      gather_store_fp8(S, kt, ms, ec, gw, lane, v, ahead ? static_cast<int>((n + 1) % kMetaSlots) : -1);
    } else if (!dry) {
      gather_issue_bf16(S, kt, ms, gw, lane);
      cp_async_wait_all();
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && !dry) {
      mbar_arrive(&S.k_full[s]);
      mbar_arrive(&S.meta_empty[ms]);
    }
    if (n == 0 && !dry) {
      query_finish(P, S, cr.b, gw, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_full);
    }
    if (n + 1 < nc && !ahead) {
      ok = mbar_wait(&S.meta_full[(n + 1) % kMetaSlots], static_cast<uint32_t>(((n + 1) / kMetaSlots) & 1),
                     &S.abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        if (lane == 0) S.abort_flag = 1;
        break;
      }
      if (fp8) gather_load_fp8(S, static_cast<int>((n + 1) % kMetaSlots), gw, lane, v, false);
    }
  }
  cp_async_wait_all();
}

// ---- warp 8, one thread: MMA1 S = Q K^T into TMEM lanes 16..31 (columns 64 (n & 1) ..
// +63: two S buffers), MMA2 O += P K into lanes 0..15 (all 512 columns; the same swizzled key
// tile read MN-major serves as V = K). MMA1 of chunk n + 1 goes out as soon as its tile and
// its S buffer are ready, ahead of MMA2 of chunk n when P of chunk n is not yet written, so
// the softmax of chunk n overlaps the tensor-core work of chunk n + 1.
__device__ void mma_role(const MqaLaunch &p, MqaSmem &S, const ChunkRange &cr, uint32_t tmem) {
  const bool f16 = fp16_operands(p);
  const uint32_t idesc1 = f16 ? idesc_f16(kH, kCh, 0, 0) : idesc_bf16(kH, kCh, 0, 0);
  const uint32_t idesc2 = f16 ? idesc_f16(kH, 256, 0, 1) : idesc_bf16(kH, 256, 0, 1);
  const uint32_t s_tmem = tmem + (16u << 16);
  const uint64_t qd = sw128_desc(smem_u32(&S.q[0][0]), 16, 1024);
  const uint64_t pd = sw128_desc(smem_u32(S.p), 16, 1024);
  // the dry pass goes once through the loop below without waiting and with every MMA and
  // commit predicated off
  const bool dry = dry_pass(S);
  const uint32_t en = dry ? 0u : 1u;
  const long long nc = dry ? (cr.lo < cr.hi ? 1 : 0) : cr.hi - cr.lo;
  // chunk m may take MMA1 once the query (chunk 0) and its tile are staged and the softmax
  // has read S of chunk m - 2
  auto s_ready = [&](long long m) {
    if (dry) return true;
    return (m > 0 || mbar_try_wait(&S.q_full, 0u)) &&
           mbar_try_wait(&S.k_full[m & 1], static_cast<uint32_t>((m >> 1) & 1)) &&
           (m < 2 || mbar_try_wait(&S.s_empty[m & 1], static_cast<uint32_t>(((m - 2) >> 1) & 1)));
  };
  auto issue_s = [&](long long m) {
    tc_fence_after();
    const uint64_t kd = sw128_desc(smem_u32(&S.k[m & 1][0][0]), 16, 1024);
    const uint32_t dt = s_tmem + 64u * static_cast<uint32_t>(m & 1);
    // (rolled by four: this loop's issue time is the tensor pipe's, and its code is fetched
    // cold once per launch)
#pragma unroll 4
    for (int kk = 0; kk < kD / 16; ++kk) {  // descriptor start advances in 16-byte units
      const uint32_t off = ((kk >> 2) * (kH * 128) + (kk & 3) * 32) >> 4;
      const uint32_t offk = ((kk >> 2) * kAtom + (kk & 3) * 32) >> 4;
      mma_bf16_if(en, dt, qd + off, kd + offk, idesc1, kk > 0 ? 1u : 0u);
    }
    mma_commit_if(en, &S.s_full[m & 1]);
  };
  long long next = 0;  // the next chunk to take MMA1
  bool ok = true;
  for (long long n = 0; ok && n < nc; ++n) {
    // P of chunk n (which needs MMA1 of chunk n); meanwhile MMA1 of chunks n and n + 1 as
    // soon as they can go
    const uint64_t t0 = globaltimer();
    uint32_t ns = 32;
    for (uint32_t i = 1;; ++i) {
      if (next <= n + 1 && next < nc && s_ready(next)) {
        issue_s(next++);
        continue;
      }
      if (dry || mbar_try_wait(&S.p_full, static_cast<uint32_t>(n & 1))) break;
      __nanosleep(ns);
      if (ns < 128) ns <<= 1;
      if ((i & 15) == 0 && (S.abort_flag || globaltimer() - t0 > kWaitLimitNs)) {
        S.abort_flag = 1;
        ok = false;
        break;
      }
    }
    if (!ok) break;
    tc_fence_after();
    const uint32_t ka = smem_u32(&S.k[n & 1][0][0]);
#pragma unroll
    for (int nh = 0; nh < 2; ++nh)
#pragma unroll
      for (int ks = 0; ks < kCh / 16; ++ks)
        mma_bf16_if(en, tmem + nh * 256, pd + ks * 2, sw128_desc(ka + nh * 4 * kAtom + ks * 2048, kAtom, 1024),
                    idesc2, (n > 0 || ks > 0) ? 1u : 0u);
    mma_commit_if(en, &S.k_empty[n & 1]);
    mma_commit_if(en, &S.o_full);
  }
  // let every MMA issued here finish (also after an abort) before anyone reads or frees the TMEM
  if (next > 0 && !dry) {
    mma_commit(&S.mma_done);
    volatile int dummy = 0;
    mbar_wait(&S.mma_done, 0u, &dummy);
  }
}

// ---- warps 0-3 (quad = warp): online softmax. Head h = 16 quad + (lane & 15): its S row is
// TMEM lane 32 quad + 16 + (lane & 15); lanes 16..31 take keys 0..31 of it, lanes 0..15
// keys 32..63 (by shuffle), and both keep the head's running state. Lanes 0..15 also own the
// head's O row (TMEM lane 32 quad + lane) for rescaling.
// Online softmax in log2 units: with z_j = x_j + ec (x_j the logit of key j), the
// accumulators hold O = sum_j 2^(z_j - R) * Krow_j and l = sum_j 2^(z_j - R) * 2^-ec, both
// from the same rounded P, in units of 2^R; R is raised lazily (only when a chunk's max z
// exceeds it by more than 8), so P stays <= 2^8 and O is rescaled rarely.
// Leaves (R, l) of each head in red_m / red_l.
__device__ void softmax_role(const MqaTcParams &P, MqaSmem &S, const ChunkRange &cr, uint32_t tmem) {
  const MqaLaunch &p = P.a;
  const int lane = threadIdx.x & 31, quad = (threadIdx.x >> 5) - kSoftWarp0;
  const int head = quad * 16 + (lane & 15);
  const bool hi = lane >= 16;  // keys 0..31 (S row owner) vs keys 32..63
  const int key0 = hi ? 0 : 32;
  const bool f16 = fp16_operands(p);
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  float R = -INFINITY, l_half = 0.f;
  long long n = 0;
  bool done = true;
  for (long long g = cr.lo; g < cr.hi; ++g, ++n) {
    const int s = static_cast<int>(n & 1);
    bool ok = true;
    if (!dry_pass(S)) {
      ok = mbar_wait(&S.k_full[s], static_cast<uint32_t>((n / 2) & 1), &S.abort_flag);
      ok = ok && mbar_wait(&S.s_full[s], static_cast<uint32_t>((n >> 1) & 1), &S.abort_flag);
    }
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      done = false;
      break;
    }
    const int ec = S.ec[s];
    // logit in log2 units of key j: acc * tau*log2(e) * qinv[h] * (fp8: 2^ec; bf16: 1)
    const float coef = P.scale_log2 * S.qinv[head] * ldexpf(1.0f, ec);
    const float fec = static_cast<float>(ec);
    tc_fence_after();
    uint32_t r0[32], r1[32];  // (lanes 0..15 read O columns here and discard them)
    tmem_ld32(lane_base + 64 * s, r0);
    tmem_ld32(lane_base + 64 * s + 32, r1);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0 && !dry_pass(S)) mbar_arrive(&S.s_empty[s]);
    const float *rs = S.rscale[s] + key0;
    float z[32];
    float mz = -INFINITY;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t other = __shfl_sync(0xFFFFFFFFu, r1[j], (lane & 15) | 16);
      const float x = __uint_as_float(hi ? r0[j] : other);
      z[j] = rs[j] != 0.f ? fmaf(x, coef, fec) : -INFINITY;
      mz = fmaxf(mz, z[j]);
    }
    mz = fmaxf(mz, __shfl_xor_sync(0xFFFFFFFFu, mz, 16));
    float Rn = R;
    if (mz > R + 8.f) Rn = mz;
    const float alpha = (Rn == R) ? 1.f : exp2f(R - Rn);  // R = -inf -> 0
    const bool need_rescale = (Rn != R) && n > 0;
    const float lsc = ldexpf(1.0f, -ec);
    float lsum = 0.f;
    uint32_t pk[16];
    const float ref = Rn == -INFINITY ? 0.f : Rn;  // a chunk with no key at all: every z is -inf
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float e0 = ex2_approx(z[j] - ref);  // z = -inf gives 0
      const float e1 = ex2_approx(z[j + 1] - ref);
      float a0, a1;
      if (f16) {
        __half2 h2 = __floats2half2_rn(e0, e1);
        pk[j / 2] = *reinterpret_cast<uint32_t *>(&h2);
        const float2 back = __half22float2(h2);
        a0 = back.x;
        a1 = back.y;
      } else {
        pk[j / 2] = pack_bf16x2(e0, e1);
        a0 = __uint_as_float(pk[j / 2] << 16);
        a1 = __uint_as_float(pk[j / 2] & 0xFFFF0000u);
      }
      lsum += a0 + a1;  // the denominator uses the rounded P, like the numerator
    }
    if (dry_pass(S)) break;  // the dry pass stops here, having changed nothing
    l_half = l_half * alpha + lsum * lsc;
    R = Rn;
    // P and O are free once MMA2 of the previous chunk completed
    ok = n == 0 || mbar_wait(&S.o_full, static_cast<uint32_t>((n - 1) & 1), &S.abort_flag);
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      done = false;
      break;
    }
    tc_fence_after();
    if (__any_sync(0xFFFFFFFFu, need_rescale)) {
      // O rows only (lanes 0..15 of the quadrant): lanes 16..31 hold S, which MMA1 of a later
      // chunk may be writing now. Thread t takes head 16 quad + t % 16, columns
      // col + 32 (t / 16) .. +31; alpha is the same in lanes t and t ^ 16.
#pragma unroll 1
      for (int col = 0; col < kD; col += 64) {
        uint32_t o[32];
        tmem_ld16x2(lane_base + col, o);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
        tmem_st16x2(lane_base + col, o);
      }
      tmem_st_wait();
    }
#pragma unroll
    for (int c = 0; c < 4; ++c)
      *reinterpret_cast<uint4 *>(S.p + sw128_offset(head, (key0 >> 3) + c)) =
          make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
    tc_fence_before();
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.p_full);
  }
  if (dry_pass(S)) return;
  const float l = l_half + __shfl_xor_sync(0xFFFFFFFFu, l_half, 16);
  if (hi) {
    S.red_m[head] = done ? R : -INFINITY;
    S.red_l[head] = done ? l : 0.f;
  }
}

__global__ void __launch_bounds__(kThreads, 1) mqa_tc_kernel(const __grid_constant__ MqaTcParams P) {
  extern __shared__ uint8_t smem_raw[];
  MqaSmem &S = *reinterpret_cast<MqaSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ float rcs[kD / 2], rsn[kD / 2];  // inverse-RoPE factors of this sequence
  const MqaLaunch &p = P.a;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_rank(), cs = cluster_size();
  const int b = blockIdx.y;

  if (tid == 0) {
    for (int i = 0; i < kMetaSlots; ++i) {
      mbar_init(&S.meta_full[i], 1);
      mbar_init(&S.meta_empty[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.k_full[i], 4);
      mbar_init(&S.k_empty[i], 1);
    }
    mbar_init(&S.q_full, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_empty[i], 4);
    }
    mbar_init(&S.p_full, 4);
    mbar_init(&S.o_full, 1);
    mbar_init(&S.mma_done, 1);
    mbar_init(&S.part_full, 1);
    S.abort_flag = 0;
    for (int w = 0; w < kThreads / 32; ++w) S.dry[w] = w == kMetaWarp ? 0 : 1;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&S.tmem_base, 512);
    tmem_relinquish();
  }
  const KeyList L = key_list(p, b, rank == 0 && tid == 0);
  const int half = p.rope_dims / 2;
  for (int i = tid; i < half; i += kThreads) rope_cos_sin(L.pos, i, p.rope_theta1, &rcs[i], &rsn[i]);
  const long long C = (L.nw + L.nsel + kCh - 1) / kCh;  // the sequence's chunks
  ChunkRange cr;
  cr.b = b;
  cr.lo = C * rank / cs;
  cr.hi = C * (rank + 1) / cs;
  pdl_wait();  // the selection (idx), the caches and the prepared query come from the kernels before
  // (the last kernel of its call: it does not release the next call's kernels early)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  // Two passes over the roles. Code that runs once per launch is fetched at the pace of a
  // cold instruction cache, several times slower than it executes. So the gather, MMA and
  // softmax warps, which would only wait while the metadata warp resolves the first chunks,
  // first go once through their long unrolled stretches over placeholder values, with no
  // waits and no effect (their S.dry flag set), then do the real pass. The metadata warp,
  // first in the chain, runs the real pass only.
#pragma unroll 1
  for (int pass = 0; pass < 2; ++pass) {
    if (warp == kMetaWarp) {
      if (pass == 1) meta_role(p, S, L, cr);
    } else if (warp >= kGatherWarp0 && warp < kGatherWarp0 + 4) {
      gather_role(P, S, cr);
    } else if (warp == kMmaWarp) {
      if (lane == 0) mma_role(p, S, cr, tmem);
    } else {
      softmax_role(P, S, cr, tmem);
    }
    __syncwarp();
    if (pass == 0 && lane == 0) S.dry[warp] = 0;
    __syncwarp();
  }

  // ---- merge of the cluster's partials. CTA q owns output columns [q Dc, (q + 1) Dc). As
  // soon as its own chunks are done, each CTA stages its O (in units of its 2^R) in rbuf as
  // one [kH][Dc] slab per owner (16-byte runs swizzled by row), bulk-copies the other
  // owners' slabs to global memory and writes its (R, l) there too; after one cluster barrier
  // each owner bulk-loads the cs - 1 slabs made for it into the freed slots and adds all cs
  // slabs with the weights 2^(R - M). Nothing crosses the cluster's shared-memory network
  // (L2 moves the slabs several times faster).
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int lcs = __ffs(static_cast<int>(cs)) - 1;  // cs is a power of two
  const int Dc = kD >> lcs, runs = Dc / 4, slab = kH * Dc;
  // warp w reads the O rows (TMEM lanes 0..15) of quadrant w % 4, columns 256 (w / 4) ..
  // +255, 64 at a time: thread t takes head 16 (w % 4) + t % 16, columns col + 32 (t / 16) .. +31
  if (warp < 8) {
    const int quad = warp & 3, h = quad * 16 + (lane & 15), col0 = (warp >> 2) * 256 + 32 * (lane >> 4);
    const bool has = cr.lo < cr.hi && !S.abort_flag;
#pragma unroll 1
    for (int c64 = 0; c64 < 256; c64 += 64) {
      uint32_t o[32];
      if (has) {
        tmem_ld16x2(tmem + (static_cast<uint32_t>(quad * 32) << 16) + (warp >> 2) * 256 + c64, o);
        tmem_ld_wait();
      }
#pragma unroll
      for (int i = 0; i < 32; i += 4) {
        const int d = col0 + c64 + i, q = d >> (9 - lcs);
        const float4 v = has ? make_float4(__uint_as_float(o[i]), __uint_as_float(o[i + 1]), __uint_as_float(o[i + 2]),
                                           __uint_as_float(o[i + 3]))
                             : make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4 *>(&S.rbuf[q * slab + h * Dc + slab_run(h, (d & (Dc - 1)) >> 2) * 4]) = v;
      }
    }
  }
  float *const part_b = P.part + static_cast<size_t>(b) * cs * (cs - 1) * slab;
  float *const red_b = P.red + static_cast<size_t>(b) * cs * 2 * kH;
  if (tid < kH) {
    red_b[(rank * 2) * kH + tid] = S.red_m[tid];
    red_b[(rank * 2 + 1) * kH + tid] = S.red_l[tid];
  }
  tc_fence_before();
  fence_proxy_async_smem();  // the staged slabs are read by the bulk copies
  __syncthreads();
  if (tid == 0 && cs > 1) {
    float *dst = part_b + static_cast<size_t>(rank) * (cs - 1) * slab;
    for (uint32_t q = 0; q < cs; ++q)
      if (q != rank) {
        bulk_store(dst, &S.rbuf[q * slab], static_cast<uint32_t>(slab * sizeof(float)));
        dst += slab;
      }
    bulk_store_wait_all();  // (also frees the slots for the loads below)
  }
  cluster_sync_all();  // every CTA's slabs and (R, l) are in global memory
  if (tid == 0 && cs > 1) {
    fence_proxy_async_global();
    mbar_arrive_expect_tx(&S.part_full, static_cast<uint32_t>((cs - 1) * slab * sizeof(float)));
    for (uint32_t src = 0; src < cs; ++src)
      if (src != rank)
        bulk_load(&S.rbuf[src * slab],
                  part_b + (static_cast<size_t>(src) * (cs - 1) + (rank < src ? rank : rank - 1)) * slab,
                  static_cast<uint32_t>(slab * sizeof(float)), &S.part_full);
  }
  if (tid < kH) {  // the weights of head tid
    float M = -INFINITY;
    for (uint32_t r = 0; r < cs; ++r) M = fmaxf(M, __ldcg(&red_b[(r * 2) * kH + tid]));
    float Ls = 0.f;
    for (uint32_t r = 0; r < cs; ++r) {
      const float m = __ldcg(&red_b[(r * 2) * kH + tid]), l = __ldcg(&red_b[(r * 2 + 1) * kH + tid]);
      const float w = m == -INFINITY ? 0.f : exp2f(m - M);
      S.wsrc[r][tid] = w;
      Ls += w * l;
    }
    S.inv_l[tid] = Ls > 0.f ? 1.f / Ls : 0.f;
    S.lse[tid] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
  }
  if (cs > 1) {
    volatile int no_abort = 0;
    if (!mbar_wait(&S.part_full, 0u, &no_abort) && tid == 0) S.abort_flag = 1;
  }
  __syncthreads();
  // CTA rank finishes its columns: the weighted sum of the cs slabs, / l, inverse RoPE, store.
  // fp8 outputs go through the freed query buffer 128 columns at a time (one [64][128] float
  // stage), each head's 128-column block quantized by one warp with its own scale.
  const bool out_fp8 = p.out_dt == DSV4_FP8E4M3;
  const int pieces = out_fp8 ? Dc / kOutBlock : 1;
  float *stage = reinterpret_cast<float *>(&S.q[0][0]);
#pragma unroll 1
  for (int pc = 0; pc < pieces; ++pc) {
    const int rope0 = kD - p.rope_dims;
    const int lruns = out_fp8 ? 5 : 7 - lcs;  // runs of 4 columns: 2^lruns (a piece of 128 for fp8)
    const int runs_here = 1 << lruns;
    for (int e = tid; e < kH * runs_here; e += kThreads) {
      const int h = e >> lruns, r4 = (e & (runs_here - 1)) + (out_fp8 ? pc * 32 : 0),
                d = static_cast<int>(rank) * Dc + r4 * 4;
      const int at = h * Dc + slab_run(h, r4) * 4;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
      for (uint32_t src = 0; src < cs; ++src) {
        const float w = S.wsrc[src][h];
        const float4 v = *reinterpret_cast<const float4 *>(&S.rbuf[src * slab + at]);
        acc.x += w * v.x;
        acc.y += w * v.y;
        acc.z += w * v.z;
        acc.w += w * v.w;
      }
      const float il = S.inv_l[h];
      float y[4] = {acc.x * il, acc.y * il, acc.z * il, acc.w * il};
#pragma unroll
      for (int u = 0; u < 4; u += 2) {
        if (d + u >= rope0) {  // rotate by -pos
          const int pi = (d + u - rope0) >> 1;
          const float c = rcs[pi], sv = rsn[pi];
          const float y0 = y[u] * c + y[u + 1] * sv, y1 = -y[u] * sv + y[u + 1] * c;
          y[u] = y0;
          y[u + 1] = y1;
        }
      }
      const size_t off = (static_cast<size_t>(b) * kH + h) * kD + d;
      if (out_fp8) {
        *reinterpret_cast<float4 *>(stage + h * kOutBlock + (r4 - pc * 32) * 4) = make_float4(y[0], y[1], y[2], y[3]);
      } else if (p.out_dt == DSV4_F32) {
        *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + off) = make_float4(y[0], y[1], y[2], y[3]);
      } else {
        *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(p.out) + off) =
            make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
      }
    }
    if (out_fp8) {
      __syncthreads();
      const int col0 = static_cast<int>(rank) * Dc + pc * kOutBlock;  // the block's first column
      for (int h = warp; h < kH; h += kThreads / 32) {
        const float4 v = *reinterpret_cast<const float4 *>(stage + h * kOutBlock + lane * 4);
        const float am = warp_max(fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
        const float scale = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
        const float inv = am > 0.f ? __fdiv_rn(448.0f, am) : 1.0f;
        const uint32_t w = static_cast<uint32_t>(float2_to_e4m3x2(__fmul_rn(v.x, inv), __fmul_rn(v.y, inv))) |
                           (static_cast<uint32_t>(float2_to_e4m3x2(__fmul_rn(v.z, inv), __fmul_rn(v.w, inv))) << 16);
        *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(p.out) + (static_cast<size_t>(b) * kH + h) * kD + col0 +
                                      lane * 4) = w;
        if (lane == 0) p.out_scales[(static_cast<size_t>(b) * kH + h) * (kD / kOutBlock) + col0 / kOutBlock] = scale;
      }
      __syncthreads();  // the stage is rewritten by the next piece
    }
  }
  if (rank == 0 && p.lse && tid < kH) p.lse[static_cast<size_t>(b) * kH + tid] = S.lse[tid];
  if (tid == 0 && S.abort_flag) report(p.d_status, DSV4_DEV_TIMEOUT);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------
// CUDA-core kernel (any dtype, D <= 1024): one CTA per (head, sequence), online softmax
// over 256-key chunks.

constexpr int kSimtChunk = 256;

__global__ void __launch_bounds__(256) mqa_simt_kernel(const MqaLaunch p, float scale_log2) {
  pdl_wait();
  extern __shared__ float sm[];
  float *qr = sm;                      // [D]
  float *xs = qr + p.D;                // [chunk]
  float *ksc = xs + kSimtChunk;        // [chunk]
  const uint8_t **kp = reinterpret_cast<const uint8_t **>(ksc + kSimtChunk);  // [chunk]
  float *red = reinterpret_cast<float *>(kp + kSimtChunk);                     // [32]
  float *ob = red + 32;                                                        // [D]
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const KeyList L = key_list(p, b, h == 0 && tid == 0);
  const int D = p.D, half = p.rope_dims / 2, rope0 = D - p.rope_dims;
  for (int d = tid; d < D; d += 256) qr[d] = load_one_f(p.q, p.q_dt, (static_cast<size_t>(b) * p.H + h) * D + d);
  __syncthreads();
  if (p.q_norm_gamma) {  // RMSNorm of the head, times gamma
    float ss = 0.f;
    for (int d = tid; d < D; d += 256) ss += qr[d] * qr[d];
    ss = block_sum(ss, red);
    const float rs = 1.0f / sqrtf(ss / static_cast<float>(D) + p.q_norm_eps);
    __syncthreads();
    for (int d = tid; d < D; d += 256) qr[d] = qr[d] * rs * p.q_norm_gamma[d];
    __syncthreads();
  }
  for (int i = tid; i < half; i += 256) {
    float c, s;
    rope_cos_sin(L.pos, i, p.rope_theta1, &c, &s);
    const float x0 = qr[rope0 + 2 * i], x1 = qr[rope0 + 2 * i + 1];
    qr[rope0 + 2 * i] = x0 * c - x1 * s;
    qr[rope0 + 2 * i + 1] = x0 * s + x1 * c;
  }
  __syncthreads();
  constexpr int kMaxPer = 4;  // D <= 1024
  float o[kMaxPer] = {0.f, 0.f, 0.f, 0.f};
  float m_run = -INFINITY, l_run = 0.f;
  const int64_t N = L.nw + L.nsel;
  for (int64_t c0 = 0; c0 < N; c0 += kSimtChunk) {
    {
      const int64_t t = c0 + tid;
      float sc = 0.f;
      const uint8_t *rp = t < N ? key_row(p, b, L, t, &sc) : nullptr;
      kp[tid] = rp;
      ksc[tid] = rp ? sc : 0.f;
    }
    __syncthreads();
    for (int i = 0; i < kSimtChunk / 8; ++i) {
      const int kk = warp * (kSimtChunk / 8) + i;
      const uint8_t *rp = kp[kk];
      float dot = 0.f;
      if (rp)
        for (int d = lane; d < D; d += 32) dot = fmaf(qr[d], load_one_f(rp, p.kv_dt, d), dot);
      dot = warp_sum(dot);
      if (lane == 0) xs[kk] = rp ? dot * ksc[kk] * scale_log2 : -INFINITY;
    }
    __syncthreads();
    float mx = -INFINITY;
    for (int i = tid; i < kSimtChunk; i += 256) mx = fmaxf(mx, xs[i]);
    mx = block_max(mx, red);
    const float m_new = fmaxf(m_run, mx);
    const float alpha = m_new == -INFINITY ? 1.f : exp2f(m_run - m_new);
    __syncthreads();
    float ls = 0.f;
    for (int i = tid; i < kSimtChunk; i += 256) {
      const float e = xs[i] == -INFINITY ? 0.f : exp2f(xs[i] - m_new);
      xs[i] = e;
      ls += e;
    }
    ls = block_sum(ls, red);
    l_run = l_run * alpha + ls;
    m_run = m_new;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kMaxPer; ++u) {
      const int d = tid + u * 256;
      if (d < D) {
        float acc = o[u] * alpha;
        for (int kk = 0; kk < kSimtChunk; ++kk) {
          const uint8_t *rp = kp[kk];
          if (rp && xs[kk] != 0.f) acc = fmaf(xs[kk] * ksc[kk], load_one_f(rp, p.kv_dt, d), acc);
        }
        o[u] = acc;
      }
    }
    __syncthreads();
  }
  const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
#pragma unroll
  for (int u = 0; u < kMaxPer; ++u) {
    const int d = tid + u * 256;
    if (d < D) ob[d] = o[u] * inv;
  }
  __syncthreads();
  for (int i = tid; i < half; i += 256) {
    float c, s;
    rope_cos_sin(L.pos, i, p.rope_theta1, &c, &s);
    const float x0 = ob[rope0 + 2 * i], x1 = ob[rope0 + 2 * i + 1];
    ob[rope0 + 2 * i] = x0 * c + x1 * s;
    ob[rope0 + 2 * i + 1] = -x0 * s + x1 * c;
  }
  __syncthreads();
  if (p.out_dt == DSV4_FP8E4M3) {  // 128-channel blocks, one scale each: a warp per block
    const int lane = tid & 31, warp = tid >> 5;
    for (int blk = warp; blk < D / kOutBlock; blk += 8) {
      float am = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) am = fmaxf(am, fabsf(ob[blk * kOutBlock + lane * 4 + u]));
      am = warp_max(am);
      const float scale = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
      const float inv = am > 0.f ? __fdiv_rn(448.0f, am) : 1.0f;
      const float *v = ob + blk * kOutBlock + lane * 4;
      const uint32_t w = static_cast<uint32_t>(float2_to_e4m3x2(__fmul_rn(v[0], inv), __fmul_rn(v[1], inv))) |
                         (static_cast<uint32_t>(float2_to_e4m3x2(__fmul_rn(v[2], inv), __fmul_rn(v[3], inv))) << 16);
      *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(p.out) + (static_cast<size_t>(b) * p.H + h) * D +
                                    blk * kOutBlock + lane * 4) = w;
      if (lane == 0) p.out_scales[(static_cast<size_t>(b) * p.H + h) * (D / kOutBlock) + blk] = scale;
    }
  } else {
    for (int d = tid; d < D; d += 256) {
      const size_t off = (static_cast<size_t>(b) * p.H + h) * D + d;
      if (p.out_dt == DSV4_F32) static_cast<float *>(p.out)[off] = ob[d];
      else static_cast<uint16_t *>(p.out)[off] = float_to_bf16_bits(ob[d]);
    }
  }
  if (p.lse && tid == 0)
    p.lse[static_cast<size_t>(b) * p.H + h] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
}

float softmax_scale_log2(const MqaLaunch &p) {
  const float s = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf(static_cast<float>(p.D));
  return s * kLog2e;
}

}  // namespace

bool mqa_uses_tensor_cores(const MqaLaunch &p) {
  return (p.kv_dt == DSV4_BF16 || p.kv_dt == DSV4_FP8E4M3) && p.D == kD && p.H == kH && p.q_dt == DSV4_BF16 &&
         p.rope_dims % 8 == 0 && p.B <= 1024;
}

// CTAs per sequence by the batch alone: as many as keep the batch within one wave of SMs
// (a power of two, at most 16). The launch may take fewer (below), never more.
static int mqa_cluster_rule(const MqaLaunch &p) {
  // (fp8 output: at most 4 CTAs, so that each owns whole 128-column blocks of the output)
  const int cap = p.out_dt == DSV4_FP8E4M3 ? kD / kOutBlock : kMaxCluster;
  int cs = 1;
  while (cs < cap && static_cast<long long>(cs) * 2 * p.B <= sm_count()) cs <<= 1;
  return cs;
}

size_t mqa_workspace_bytes(const MqaLaunch &p) {
  if (!mqa_uses_tensor_cores(p)) return 0;
  const size_t cs = static_cast<size_t>(mqa_cluster_rule(p));
  return align_up(static_cast<size_t>(p.B) * kH * kD * sizeof(uint16_t), 256) +
         align_up(static_cast<size_t>(p.B) * kH * sizeof(float), 256) +
         align_up(static_cast<size_t>(p.B) * kMaxCluster * 2 * kH * sizeof(float), 256) +
         align_up(static_cast<size_t>(p.B) * (cs - 1) * kH * kD * sizeof(float), 256);
}

// CTAs per sequence: the rule above, at most 8 where the device cannot co-schedule 16 of
// these CTAs
static int mqa_cluster(const MqaLaunch &p, size_t smem) {
  int cs = mqa_cluster_rule(p);
  if (cs > 8) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(cs), static_cast<unsigned>(p.B));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(cs);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaFuncSetAttribute(mqa_tc_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, mqa_tc_kernel, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      cs = 8;
    }
  }
  return cs;
}

static MqaTcParams tc_params(const MqaLaunch &p0, void *ws) {
  MqaTcParams P;
  P.a = p0;
  P.a.rope_theta1 = rope_theta1(p0.rope_base, p0.rope_dims);
  P.scale_log2 = softmax_scale_log2(P.a);
  char *w = static_cast<char *>(ws);
  P.qp = reinterpret_cast<uint16_t *>(w);
  w += align_up(static_cast<size_t>(p0.B) * kH * kD * sizeof(uint16_t), 256);
  P.qinv = reinterpret_cast<float *>(w);
  w += align_up(static_cast<size_t>(p0.B) * kH * sizeof(float), 256);
  P.red = reinterpret_cast<float *>(w);
  w += align_up(static_cast<size_t>(p0.B) * kMaxCluster * 2 * kH * sizeof(float), 256);
  P.part = reinterpret_cast<float *>(w);
  return P;
}

cudaError_t launch_mqa_query(const MqaLaunch &p, void *ws, cudaStream_t st) {
  if (!mqa_uses_tensor_cores(p)) return cudaSuccess;
  return launch_pdl(mqa_query_kernel, dim3(p.B, kH / 8), dim3(128), 0, st, 1, tc_params(p, ws));
}

cudaError_t launch_mqa_attention(const MqaLaunch &p0, void *ws, cudaStream_t st) {
  MqaLaunch p = p0;
  p.rope_theta1 = rope_theta1(p.rope_base, p.rope_dims);
  if (mqa_uses_tensor_cores(p)) {
    const MqaTcParams P = tc_params(p0, ws);
    const size_t smem = sizeof(MqaSmem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(mqa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int cs = mqa_cluster(p, smem);
    return launch_pdl(mqa_tc_kernel, dim3(static_cast<unsigned>(cs), static_cast<unsigned>(p.B)), dim3(kThreads),
                      smem, st, cs, P);
  }
  const size_t smem = (2 * static_cast<size_t>(p.D) + 2 * kSimtChunk + 32) * sizeof(float) +
                      kSimtChunk * sizeof(void *) + 16;
  cudaError_t e = cudaFuncSetAttribute(mqa_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(mqa_simt_kernel, dim3(p.H, p.B), dim3(256), smem, st, 1, p, softmax_scale_log2(p));
}

cudaError_t launch_mqa(const MqaLaunch &p, void *ws, cudaStream_t st) {
  const cudaError_t e = launch_mqa_query(p, ws, st);
  if (e != cudaSuccess) return e;
  return launch_mqa_attention(p, ws, st);
}

}  // namespace dsv4
