// Shared-K/V multi-query attention of one decode query per sequence, with the query
// rotated by RoPE_pos and the output rotated back by -pos (steps (3) and (4) of the decode
// method; vLLM "four moves": shared K/V + inverse RoPE, sparse attention over compressed
// tokens united with a short sliding window; SGLang "Shadow radix": SWA-128 + C4 top-512
// or C128 dense).
//
// Keys of sequence s (V = K): window positions max(0,p-W+1)..p, then the selected entries
// idx[s][0..k) (C4) or all visible entries (C128).
//
// Tensor-core path (bf16/fp8 caches, D = 512, H = 64): split-K over 64-key chunks of the
// flattened (sequence, chunk) space, one persistent CTA per SM. Per chunk:
//   gather: 64 key rows (16-byte loads; fp8 -> bf16 is exact) into a 128B-swizzled tile,
//   MMA1:   S[64 heads x 64 keys] = Q K^T   (tcgen05 kind::f16, M = 64, accum at TMEM lane 16)
//   softmax per head in one thread (the S row sits in that thread's TMEM lane), online
//           with a lazy reference max (rescale only when the max grows by > 2^8),
//           P' = exp2(x - m) * scale_j as bf16 (the fp8 row scale folded into P),
//   MMA2:   O[64 x 512] += P' K               (M = 64, N = 256 x 2, K MN-major from the
//           same swizzled tile, accum at TMEM lane 0, all 512 columns).
// The gather of chunk i+1 overlaps MMA1 of chunk i. Each (CTA, sequence) segment writes
// an unnormalized partial (O, m, l); a merge kernel combines partials with their
// log-sum-exp weights, applies the inverse RoPE and stores the output.
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

// prefix[b] = number of 64-key chunks of sequences 0..b-1, prefix[B] = total; computed by
// every thread of the CTA (contiguous slices of sequences, then a two-level shuffle scan of
// the slice sums). red: 32 scratch values. blockDim.x is a multiple of 32.
__device__ void chunk_prefix(const MqaLaunch &p, long long *prefix, long long *red, bool report_it) {
  const int nt = blockDim.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int lo = static_cast<int>((static_cast<long long>(p.B) * t) / nt);
  const int hi = static_cast<int>((static_cast<long long>(p.B) * (t + 1)) / nt);
  long long mine = 0;
  for (int b = lo; b < hi; ++b) {
    const KeyList L = key_list(p, b, report_it);
    const long long c = (L.nw + L.nsel + 63) / 64;
    prefix[b] = c;
    mine += c;
  }
  long long v = mine;  // inclusive scan within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long u = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    long long w = lane < (nt >> 5) ? red[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long u = __shfl_up_sync(0xFFFFFFFFu, w, o);
      if (lane >= o) w += u;
    }
    red[lane] = w;
  }
  __syncthreads();
  long long acc = v - mine + (warp > 0 ? red[warp - 1] : 0);
  if (t == nt - 1) prefix[p.B] = acc + mine;
  for (int b = lo; b < hi; ++b) {
    const long long c = prefix[b];
    prefix[b] = acc;
    acc += c;
  }
  __syncthreads();
}

__device__ __forceinline__ int find_seq(const long long *prefix, int B, long long g) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// ------------------------------------------------------------------------------------
// tensor-core kernel

constexpr int kH = 64, kD = 512, kCh = 64;
constexpr int kAtom = kCh * 128;  // one 64-dim column block of a 64-row tile: 8 KB
constexpr int kMetaSlots = 4;     // chunks whose key metadata is resolved ahead
// roles: warps 0-3 softmax + output (TMEM lane quadrant = warp), warps 4-7 gather, warp 8
// MMA issue (and TMEM allocation), warp 9 key metadata
constexpr int kSoftWarp0 = 0, kGatherWarp0 = 4, kMmaWarp = 8, kMetaWarp = 9;
constexpr int kThreads = 320;

struct alignas(1024) MqaSmem {
  uint8_t q[kD / 64][kH * 128];      // 64 KB, K-major SW128, 8 atoms of 64 dims
  uint8_t k[2][kD / 64][kCh * 128];  // 2 x 64 KB key tiles (stage = chunk parity)
  uint8_t p[kH * 128];               // 8 KB: P[64 heads][64 keys], K-major SW128
  const uint8_t *mrow[kMetaSlots][kCh];  // row address of each key of a chunk (nullptr: none)
  float mscale[kMetaSlots][kCh];         // its row scale
  float rscale[2][kCh];                  // row scale per key of a staged tile (0: no key)
  int ec[2];                             // tile exponent: K rows hold code * scale * 2^-ec
  float qinv[2][kH];                     // 2^-e of the per-head query scale, by segment parity
  uint64_t meta_full[kMetaSlots], meta_empty[kMetaSlots];
  uint64_t k_full[2], k_empty[2], q_full, q_empty, s_full, s_empty, p_full, o_full, o_empty;
  uint32_t tmem_base;
  int abort_flag;
};

struct MqaTcParams {
  MqaLaunch a;
  float scale_log2;
  float *part_o;   // [B + G][H][D]
  float *part_ml;  // [B + G][H][2]
  uint16_t *qp;    // [B][H][D] query rotated by RoPE_pos, fp16 (scaled per head) or bf16
  float *qinv;     // [B][H] 2^-e undoing the per-head scale (1 for bf16)
};

// Operands of the two MMAs. fp8 caches: fp16 (e4m3 -> fp16 is exact, and fp16 keeps 11
// significand bits of the rotated query and of P); bf16 caches: bf16.
__device__ __forceinline__ bool fp16_operands(const MqaLaunch &p) { return p.kv_dt == DSV4_FP8E4M3; }

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// where chunk g sits: its sequence, and whether it opens / closes this CTA's run of it
struct ChunkPos {
  int b;
  bool first, last;
};
__device__ __forceinline__ ChunkPos chunk_pos(const long long *prefix, int B, long long g, long long c0,
                                              long long c1) {
  ChunkPos c;
  c.b = find_seq(prefix, B, g);
  c.first = g == c0 || prefix[c.b] == g;
  c.last = g + 1 == c1 || prefix[c.b + 1] == g + 1;
  return c;
}

// ---- warp 9: row address and scale of every key of up to kMetaSlots chunks at a time.
// The idx -> block table -> scale chain is staged over all keys of the batch, so its three
// memory latencies are paid once per batch.
__device__ void meta_role(const MqaLaunch &p, MqaSmem &S, const long long *prefix, long long c0, long long c1) {
  const int lane = threadIdx.x & 31;
  const int per_page = DSV4_PAGE_POSITIONS / p.m;
  const size_t esz = dtype_size(p.kv_dt);
  constexpr int kKeys = kMetaSlots * 2;  // keys per lane per batch
  for (long long g0 = c0; g0 < c1; g0 += kMetaSlots) {
    const int nb = static_cast<int>(c1 - g0 < kMetaSlots ? c1 - g0 : kMetaSlots);
    bool ok = true;
    for (int i = 0; i < nb; ++i) {
      const long long n = g0 + i - c0;
      if (n >= kMetaSlots && lane == 0 &&
          !mbar_wait(&S.meta_empty[n % kMetaSlots], static_cast<uint32_t>((n / kMetaSlots - 1) & 1), &S.abort_flag))
        ok = false;
    }
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      return;
    }
    int bc[kMetaSlots];
    KeyList Lc[kMetaSlots];
#pragma unroll
    for (int i = 0; i < kMetaSlots; ++i) {
      bc[i] = i < nb ? find_seq(prefix, p.B, g0 + i) : 0;
      if (i < nb) Lc[i] = key_list(p, bc[i], false);
    }
    int bseq[kKeys];
    int64_t j[kKeys];  // >= 0: entry index; -1: none; -2 - slot: window ring slot
    int32_t page[kKeys];
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {  // stage 1: key list position -> entry index (idx load)
      const int i = u >> 1;
      j[u] = -1;
      bseq[u] = 0;
      if (i < nb) {
        const int b = bc[i];
        const KeyList &L = Lc[i];
        const int64_t t = (g0 + i - prefix[b]) * kCh + lane + 32 * (u & 1);
        bseq[u] = b;
        if (t < L.nw) {
          const int64_t pw = L.pos - L.nw + 1 + t;
          j[u] = -2 - (static_cast<int64_t>(b) * p.W + pw % p.W);
        } else if (t - L.nw < L.nsel) {
          const int64_t uu = t - L.nw;
          int64_t e = uu;
          if (p.idx) {
            e = p.idx[static_cast<size_t>(b) * p.k + uu];
            if (e >= L.n_entries) {
              report(p.d_status, DSV4_DEV_BAD_INDEX);
              e = -1;
            }
          }
          j[u] = e < 0 ? -1 : e;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {  // stage 2: entry -> physical page (block table load)
      page[u] = -1;
      if (j[u] >= 0) {
        page[u] = p.block_table[static_cast<size_t>(bseq[u]) * p.max_blocks + j[u] / per_page];
        if (page[u] < 0 || page[u] >= p.num_pages) {
          report(p.d_status, DSV4_DEV_BAD_PAGE);
          page[u] = -1;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kKeys; ++u) {  // stage 3: row address and scale
      const int i = u >> 1;
      if (i >= nb) continue;
      const uint8_t *rp = nullptr;
      float sc = 0.f;
      if (j[u] <= -2) {
        const size_t slot = static_cast<size_t>(-2 - j[u]);
        rp = static_cast<const uint8_t *>(p.ring_rows) + slot * p.D * esz;
        sc = p.kv_dt == DSV4_FP8E4M3 ? p.ring_scales[slot] : 1.0f;
      } else if (page[u] >= 0) {
        const size_t row = static_cast<size_t>(page[u]) * per_page + static_cast<size_t>(j[u] % per_page);
        rp = static_cast<const uint8_t *>(p.pages) + row * p.D * esz;
        sc = p.kv_dt == DSV4_FP8E4M3 ? p.scales[row] : 1.0f;
      }
      const int slot = static_cast<int>((g0 + i - c0) % kMetaSlots);
      S.mrow[slot][lane + 32 * (u & 1)] = rp;
      S.mscale[slot][lane + 32 * (u & 1)] = rp ? sc : 0.f;
    }
    __syncwarp();
    if (lane == 0)
      for (int i = 0; i < nb; ++i) mbar_arrive(&S.meta_full[(g0 + i - c0) % kMetaSlots]);
  }
}

// ---- the query of every sequence, rotated by RoPE_pos once: bf16, or fp16 scaled per
// head by a power of two (qinv undoes it in the logits) so that |q| < 2^14 whatever the
// input range. grid (B), 256 threads: thread t owns dims 128 (t & 3) .. +127 of head t / 4.
// It reads only the caller's query and writes only qp/qinv, which nothing before it on the
// stream reads, so it runs before its pdl_wait(), beside the kernel before it.
__global__ void __launch_bounds__(256) mqa_query_kernel(const MqaTcParams P) {
  const MqaLaunch &p = P.a;
  __shared__ float cs[kD / 2], sn[kD / 2];
  const int b = blockIdx.x, t = threadIdx.x, h = t >> 2, d0 = (t & 3) * 128;
  const bool f16 = fp16_operands(p);
  const int half = p.rope_dims / 2, rope0 = kD - p.rope_dims;
  const int64_t pos = p.pos[b];
  for (int i = t; i < half; i += 256) rope_cos_sin(pos, i, p.rope_theta1, &cs[i], &sn[i]);
  const uint4 *src = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(p.q) +
                                                     (static_cast<size_t>(b) * kH + h) * kD + d0);
  uint4 raw[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) raw[i] = __ldg(src + i);
  __syncthreads();
  auto rotated = [&](int i, float *x) {  // the 8 values of run i, rotated where they are rope dims
    const uint32_t v[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      x[2 * u] = __uint_as_float(v[u] << 16);
      x[2 * u + 1] = __uint_as_float(v[u] & 0xFFFF0000u);
      const int d = d0 + i * 8 + 2 * u;
      if (d >= rope0) {
        const float c = cs[(d - rope0) >> 1], sv = sn[(d - rope0) >> 1];
        const float x0 = x[2 * u], x1 = x[2 * u + 1];
        x[2 * u] = x0 * c - x1 * sv;
        x[2 * u + 1] = x0 * sv + x1 * c;
      }
    }
  };
  float qs = 1.0f, qi = 1.0f;
  if (f16) {
    float am = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float x[8];
      rotated(i, x);
#pragma unroll
      for (int u = 0; u < 8; ++u) am = fmaxf(am, fabsf(x[u]));
    }
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 1));
    am = fmaxf(am, __shfl_xor_sync(0xFFFFFFFFu, am, 2));
    int e = 0;
    if (am > 0.f) frexpf(am, &e);  // am < 2^e
    qi = am > 0.f ? ldexpf(1.0f, e - 14) : 1.0f;
    qs = am > 0.f ? ldexpf(1.0f, 14 - e) : 1.0f;
  }
  uint4 *dst = reinterpret_cast<uint4 *>(P.qp + (static_cast<size_t>(b) * kH + h) * kD + d0);
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    float x[8];
    rotated(i, x);
    dst[i] = f16 ? make_uint4(pack_f16x2(x[0] * qs, x[1] * qs), pack_f16x2(x[2] * qs, x[3] * qs),
                              pack_f16x2(x[4] * qs, x[5] * qs), pack_f16x2(x[6] * qs, x[7] * qs))
                 : make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                              pack_bf16x2(x[6], x[7]));
  }
  if ((t & 3) == 0) P.qinv[static_cast<size_t>(b) * kH + h] = qi;
  pdl_wait();
  pdl_launch_dependents();
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

__device__ __forceinline__ void query_finish(const MqaTcParams &P, MqaSmem &S, int b, int par, int gw, int lane) {
  if (lane < 16) S.qinv[par][gw * 16 + lane] = P.qinv[static_cast<size_t>(b) * kH + gw * 16 + lane];
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

__device__ __forceinline__ void gather_load_fp8(const MqaSmem &S, int ms, int gw, int lane, uint4 (&v)[16]) {
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const uint8_t *rp = S.mrow[ms][gw * 16 + rr];
    v[rr] = rp ? __ldg(reinterpret_cast<const uint4 *>(rp + lane * 16)) : make_uint4(0, 0, 0, 0);
  }
}

__device__ __forceinline__ void gather_store_fp8(MqaSmem &S, uint8_t *kt, int ms, int ec, int gw, int lane, const uint4 (&v)[16]) {
  const int atom = lane >> 2, c0 = (lane & 3) * 2;
#pragma unroll
  for (int rr = 0; rr < 16; ++rr) {
    const int row = gw * 16 + rr;
    const __half2 sc2 = __float2half2_rn(ldexpf(S.mscale[ms][row], -ec));
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
  }
}

__device__ void gather_role(const MqaTcParams &P, MqaSmem &S, const long long *prefix, long long c0, long long c1) {
  const MqaLaunch &p = P.a;
  const int lane = threadIdx.x & 31, gw = (threadIdx.x >> 5) - kGatherWarp0;
  const bool fp8 = p.kv_dt == DSV4_FP8E4M3;
  int seg = -1;
  for (long long g = c0; g < c1; ++g) {
    const long long n = g - c0;
    const int s = static_cast<int>(n & 1), ms = static_cast<int>(n % kMetaSlots);
    const ChunkPos cp = chunk_pos(prefix, p.B, g, c0, c1);
    bool ok = mbar_wait(&S.meta_full[ms], static_cast<uint32_t>((n / kMetaSlots) & 1), &S.abort_flag);
    if (ok && cp.first) {
      ++seg;
      if (seg >= 1) ok = mbar_wait(&S.q_empty, static_cast<uint32_t>((seg - 1) & 1), &S.abort_flag);
      if (ok) query_issue(P, S, cp.b, gw, lane);
    }
    if (ok && n >= 2) ok = mbar_wait(&S.k_empty[s], static_cast<uint32_t>((n / 2 - 1) & 1), &S.abort_flag);
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      break;
    }
    // the query copy (if any) and the key rows are in flight together; the tile is finished
    // first, then the query
    uint8_t *kt = &S.k[s][0][0];
    // chunk exponent (every warp derives the same one) and the scales softmax reads
    const float smax = warp_max(fmaxf(S.mscale[ms][lane], S.mscale[ms][lane + 32]));
    int ec = 0;
    if (fp8) frexpf(smax, &ec);  // largest scale = f * 2^ec, f in [0.5, 1)
    if (lane < 16) S.rscale[s][gw * 16 + lane] = S.mscale[ms][gw * 16 + lane];
    if (gw == 0 && lane == 0) S.ec[s] = ec;
    if (fp8) {
      uint4 v[16];
      gather_load_fp8(S, ms, gw, lane, v);
      gather_store_fp8(S, kt, ms, ec, gw, lane, v);
    } else {
      gather_issue_bf16(S, kt, ms, gw, lane);
      cp_async_wait_all();
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      mbar_arrive(&S.k_full[s]);
      mbar_arrive(&S.meta_empty[ms]);
    }
    if (cp.first) {
      query_finish(P, S, cp.b, seg & 1, gw, lane);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_full);
    }
  }
  cp_async_wait_all();
}

// ---- warp 8, one thread: MMA1 S = Q K^T into TMEM lanes 16..31, MMA2 O += P K into lanes
// 0..15 (all 512 columns; the same swizzled key tile read MN-major serves as V = K).
__device__ void mma_role(const MqaLaunch &p, MqaSmem &S, const long long *prefix, long long c0, long long c1,
                         uint32_t tmem) {
  const bool f16 = fp16_operands(p);
  const uint32_t idesc1 = f16 ? idesc_f16(kH, kCh, 0, 0) : idesc_bf16(kH, kCh, 0, 0);
  const uint32_t idesc2 = f16 ? idesc_f16(kH, 256, 0, 1) : idesc_bf16(kH, 256, 0, 1);
  const uint32_t s_tmem = tmem + (16u << 16);
  int seg = -1;
  long long n = 0;
  for (long long g = c0; g < c1; ++g, ++n) {
    const int s = static_cast<int>(n & 1);
    const ChunkPos cp = chunk_pos(prefix, p.B, g, c0, c1);
    if (cp.first) {
      ++seg;
      if (!mbar_wait(&S.q_full, static_cast<uint32_t>(seg & 1), &S.abort_flag)) break;
    }
    if (!mbar_wait(&S.k_full[s], static_cast<uint32_t>((n / 2) & 1), &S.abort_flag)) break;
    if (n >= 1 && !mbar_wait(&S.s_empty, static_cast<uint32_t>((n - 1) & 1), &S.abort_flag)) break;
    tc_fence_after();
    const uint32_t qa = smem_u32(&S.q[0][0]), ka = smem_u32(&S.k[s][0][0]);
#pragma unroll 4
    for (int kk = 0; kk < kD / 16; ++kk) {
      const uint32_t off = (kk >> 2) * (kH * 128) + (kk & 3) * 32;
      const uint32_t offk = (kk >> 2) * kAtom + (kk & 3) * 32;
      mma_bf16(s_tmem, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + offk, 16, 1024), idesc1, kk > 0 ? 1u : 0u);
    }
    mma_commit(&S.s_full);
    if (cp.last) mma_commit(&S.q_empty);
    if (!mbar_wait(&S.p_full, static_cast<uint32_t>(n & 1), &S.abort_flag)) break;
    if (cp.first && seg >= 1 && !mbar_wait(&S.o_empty, static_cast<uint32_t>((seg - 1) & 1), &S.abort_flag)) break;
    tc_fence_after();
    const uint32_t pa = smem_u32(S.p);
#pragma unroll
    for (int nh = 0; nh < 2; ++nh)
#pragma unroll
      for (int ks = 0; ks < kCh / 16; ++ks)
        mma_bf16(tmem + nh * 256, sw128_desc(pa + ks * 32, 16, 1024),
                 sw128_desc(ka + nh * 4 * kAtom + ks * 2048, kAtom, 1024), idesc2,
                 (!cp.first || ks > 0) ? 1u : 0u);
    mma_commit(&S.k_empty[s]);
    mma_commit(&S.o_full);
  }
  // let the last MMAs finish before the CTA frees its TMEM
  if (n > 0) {
    volatile int dummy = 0;
    mbar_wait(&S.o_full, static_cast<uint32_t>((n - 1) & 1), &dummy);
  }
}

// ---- warps 0-3 (quad = warp): online softmax and the partial output. Head h = 16 quad +
// (lane & 15): its S row is TMEM lane 32 quad + 16 + (lane & 15); lanes 16..31 take keys
// 0..31 of it, lanes 0..15 keys 32..63 (by shuffle), and both keep the head's running state.
// Lanes 0..15 also own the head's O row (TMEM lane 32 quad + lane) for rescaling and output.
// Online softmax in log2 units: with z_j = x_j + ec (x_j the logit of key j), the
// accumulators hold O = sum_j 2^(z_j - R) * Krow_j and l = sum_j 2^(z_j - R) * 2^-ec, both
// from the same rounded P, in units of 2^R; R is raised lazily (only when a chunk's max z
// exceeds it by more than 8), so P stays <= 2^8 and O is rescaled rarely.
__device__ void softmax_role(const MqaTcParams &P, MqaSmem &S, const long long *prefix, long long c0, long long c1,
                             uint32_t tmem) {
  const MqaLaunch &p = P.a;
  const int lane = threadIdx.x & 31, quad = (threadIdx.x >> 5) - kSoftWarp0;
  const int head = quad * 16 + (lane & 15);
  const bool hi = lane >= 16;            // keys 0..31 (S row owner) vs keys 32..63
  const int key0 = hi ? 0 : 32;
  const bool f16 = fp16_operands(p);
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  float R = -INFINITY, l_half = 0.f;
  int seg = -1;
  long long n = 0;
  for (long long g = c0; g < c1; ++g, ++n) {
    const int s = static_cast<int>(n & 1);
    const ChunkPos cp = chunk_pos(prefix, p.B, g, c0, c1);
    if (cp.first) {
      ++seg;
      R = -INFINITY;
      l_half = 0.f;
    }
    bool ok = mbar_wait(&S.k_full[s], static_cast<uint32_t>((n / 2) & 1), &S.abort_flag);
    ok = ok && mbar_wait(&S.s_full, static_cast<uint32_t>(n & 1), &S.abort_flag);
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      break;
    }
    // read the query scale before releasing S: once S is free the query of a later segment
    // (same parity) may be written
    const int ec = S.ec[s];
    // logit in log2 units of key j: acc * tau*log2(e) * qinv[h] * (fp8: 2^ec; bf16: 1)
    const float coef = P.scale_log2 * S.qinv[seg & 1][head] * ldexpf(1.0f, ec);
    const float fec = static_cast<float>(ec);
    tc_fence_after();
    uint32_t r0[32], r1[32];
    tmem_ld32(lane_base + 0, r0);
    tmem_ld32(lane_base + 32, r1);
    tmem_ld_wait();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(&S.s_empty);
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
    const bool need_rescale = (Rn != R) && !cp.first;
    const float lsc = ldexpf(1.0f, -ec);
    float lsum = 0.f;
    uint32_t pk[16];
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      const float e0 = z[j] == -INFINITY ? 0.f : exp2f(z[j] - Rn);
      const float e1 = z[j + 1] == -INFINITY ? 0.f : exp2f(z[j + 1] - Rn);
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
    l_half = l_half * alpha + lsum * lsc;
    R = Rn;
    // P and O are free once MMA2 of the previous chunk completed
    ok = n == 0 || mbar_wait(&S.o_full, static_cast<uint32_t>((n - 1) & 1), &S.abort_flag);
    if (!__all_sync(0xFFFFFFFFu, ok)) {
      if (lane == 0) S.abort_flag = 1;
      break;
    }
    tc_fence_after();
    if (__any_sync(0xFFFFFFFFu, need_rescale)) {
#pragma unroll 1
      for (int col = 0; col < kD; col += 32) {
        uint32_t o[32];
        tmem_ld32(lane_base + col, o);
        tmem_ld_wait();
        if (!hi) {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
        }
        tmem_st32(lane_base + col, o);
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
    if (cp.last) {
      const float l = l_half + __shfl_xor_sync(0xFFFFFFFFu, l_half, 16);
      ok = mbar_wait(&S.o_full, static_cast<uint32_t>(n & 1), &S.abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) {
        if (lane == 0) S.abort_flag = 1;
        break;
      }
      tc_fence_after();
      const size_t slot = static_cast<size_t>(cp.b) + blockIdx.x;
      if (hi) {
        float *ml = P.part_ml + (slot * kH + head) * 2;
        ml[0] = R;
        ml[1] = l;
      }
      float *po = P.part_o + (slot * kH + head) * kD;
#pragma unroll 1
      for (int col = 0; col < kD; col += 128) {  // four loads in flight per wait
        uint32_t o[4][32];
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_ld32(lane_base + col + 32 * c, o[c]);
        tmem_ld_wait();
        if (!hi) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              __stcg(reinterpret_cast<float4 *>(po + col + 32 * c + i),
                     make_float4(__uint_as_float(o[c][i]), __uint_as_float(o[c][i + 1]), __uint_as_float(o[c][i + 2]),
                                 __uint_as_float(o[c][i + 3])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.o_empty);
    }
  }
}

__global__ void __launch_bounds__(kThreads, 1) mqa_tc_kernel(const __grid_constant__ MqaTcParams P) {
  extern __shared__ uint8_t smem_raw[];
  MqaSmem &S = *reinterpret_cast<MqaSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const MqaLaunch &p = P.a;
  long long *prefix = reinterpret_cast<long long *>(&S + 1);  // [B + 1] chunks before sequence b
  const int tid = threadIdx.x, warp = tid >> 5;

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
    mbar_init(&S.q_empty, 1);
    mbar_init(&S.s_full, 1);
    mbar_init(&S.s_empty, 4);
    mbar_init(&S.p_full, 4);
    mbar_init(&S.o_full, 1);
    mbar_init(&S.o_empty, 4);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&S.tmem_base, 512);
    tmem_relinquish();
  }
  chunk_prefix(p, prefix, prefix + p.B + 1, blockIdx.x == 0);
  pdl_wait();  // the selection (idx) and the caches come from the kernels before
  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const long long T = prefix[p.B], G = gridDim.x;
  const long long c0 = (T * blockIdx.x) / G, c1 = (T * (blockIdx.x + 1)) / G;

  if (warp == kMetaWarp) meta_role(p, S, prefix, c0, c1);
  else if (warp >= kGatherWarp0 && warp < kGatherWarp0 + 4) gather_role(P, S, prefix, c0, c1);
  else if (warp == kMmaWarp) {
    if ((tid & 31) == 0) mma_role(p, S, prefix, c0, c1, tmem);
  } else softmax_role(P, S, prefix, c0, c1, tmem);

  if (tid == 0 && S.abort_flag) report(p.d_status, DSV4_DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the partials of every sequence, inverse RoPE, store. grid (B, H / 8), 256 threads:
// warp w owns head h0 + w for the weights; for the sum every thread owns 4 float4 columns
// of the CTA's 8 heads and keeps their loads of several partials in flight together.
__global__ void __launch_bounds__(256) mqa_merge_kernel(const MqaTcParams P, int grid_ctas) {
  const MqaLaunch &p = P.a;
  __shared__ int warp_cnt[8];
  __shared__ float cs[kD / 2], sn[kD / 2];
  __shared__ float inv_l[8], lse_s[8];
  extern __shared__ __align__(16) uint8_t dyn[];
  float *wgt = reinterpret_cast<float *>(dyn);                                  // [grid][8] weight
  float *lv = wgt + static_cast<size_t>(grid_ctas) * 8;                         // [grid][8] partial sum
  int *cta = reinterpret_cast<int *>(lv + static_cast<size_t>(grid_ctas) * 8);  // [grid]
  long long *prefix = reinterpret_cast<long long *>(cta + ((grid_ctas + 1) & ~1));  // [B + 1]
  long long *red = prefix + p.B + 1;                                             // [blockDim]
  const int b = blockIdx.x, h0 = blockIdx.y * 8, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const KeyList L = key_list(p, b, false);
  const int half = p.rope_dims / 2;
  for (int i = tid; i < half; i += 256) rope_cos_sin(L.pos, i, p.rope_theta1, &cs[i], &sn[i]);
  chunk_prefix(p, prefix, red, false);
  // the CTAs of the main kernel whose (non-empty) chunk range meets this sequence, in
  // order; with fewer chunks than CTAs some ranges are empty and those CTAs wrote nothing
  const long long acc = prefix[p.B], mine = prefix[b], cnt = prefix[b + 1] - prefix[b];
  int n = 0;
  for (int c0 = 0; c0 < grid_ctas; c0 += 256) {
    const int c = c0 + tid;
    bool hit = false;
    if (c < grid_ctas && cnt > 0) {
      const long long a0 = (acc * c) / grid_ctas, a1 = (acc * (c + 1)) / grid_ctas;
      hit = a0 < mine + cnt && a1 > mine && a1 > a0;
    }
    const unsigned bal = __ballot_sync(0xFFFFFFFFu, hit);
    if (lane == 0) warp_cnt[warp] = __popc(bal);
    __syncthreads();
    int off = n;
    for (int w = 0; w < warp; ++w) off += warp_cnt[w];
    if (hit) cta[off + __popc(bal & ((1u << lane) - 1u))] = c;
    for (int w = 0; w < 8; ++w) n += warp_cnt[w];
    __syncthreads();
  }
  const int np = n;
  pdl_wait();  // the partials come from the kernel before
  pdl_launch_dependents();
  for (int j = tid; j < np * 8; j += 256) {
    const size_t slot = static_cast<size_t>(b) + cta[j >> 3];
    const float2 ml = *reinterpret_cast<const float2 *>(P.part_ml + (slot * kH + h0 + (j & 7)) * 2);
    wgt[j] = ml.x;
    lv[j] = ml.y;
  }
  __syncthreads();
  {  // weights of head h0 + warp: 2^(m_i - M), M the largest partial reference
    float M = -INFINITY;
    for (int i = lane; i < np; i += 32) M = fmaxf(M, wgt[i * 8 + warp]);
    M = warp_max(M);
    float Ls = 0.f;
    for (int i = lane; i < np; i += 32) {
      const float mi = wgt[i * 8 + warp];
      const float w = (mi == -INFINITY) ? 0.f : exp2f(mi - M);
      wgt[i * 8 + warp] = w;
      Ls += w * lv[i * 8 + warp];
    }
    Ls = warp_sum(Ls);
    if (lane == 0) {
      inv_l[warp] = Ls > 0.f ? 1.f / Ls : 0.f;
      lse_s[warp] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
    }
  }
  __syncthreads();
  constexpr int kPer = 8 * kD / 4 / 256;  // float4 columns per thread (4)
  float4 o[kPer];
#pragma unroll
  for (int q = 0; q < kPer; ++q) o[q] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int i = 0; i < np; ++i) {
    const size_t slot = static_cast<size_t>(b) + cta[i];
    const float *base = P.part_o + (slot * kH + h0) * kD;
    float4 v[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) v[q] = __ldcs(reinterpret_cast<const float4 *>(base) + q * 256 + tid);
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const float w = wgt[i * 8 + (q * 256 + tid) / (kD / 4)];
      o[q].x = fmaf(w, v[q].x, o[q].x);
      o[q].y = fmaf(w, v[q].y, o[q].y);
      o[q].z = fmaf(w, v[q].z, o[q].z);
      o[q].w = fmaf(w, v[q].w, o[q].w);
    }
  }
  const int rope0 = kD - p.rope_dims;
#pragma unroll
  for (int q = 0; q < kPer; ++q) {
    const int e = q * 256 + tid, hh = e / (kD / 4), d = (e % (kD / 4)) * 4, h = h0 + hh;
    float y[4] = {o[q].x * inv_l[hh], o[q].y * inv_l[hh], o[q].z * inv_l[hh], o[q].w * inv_l[hh]};
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      if (d + u >= rope0) {  // rotate by -pos
        const int pi = (d + u - rope0) >> 1;
        const float c = cs[pi], sv = sn[pi];
        const float y0 = y[u] * c + y[u + 1] * sv, y1 = -y[u] * sv + y[u + 1] * c;
        y[u] = y0;
        y[u + 1] = y1;
      }
    }
    const size_t off = (static_cast<size_t>(b) * kH + h) * kD + d;
    if (p.out_dt == DSV4_F32) {
      *reinterpret_cast<float4 *>(static_cast<float *>(p.out) + off) = make_float4(y[0], y[1], y[2], y[3]);
    } else {
      *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(p.out) + off) =
          make_uint2(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]));
    }
  }
  if (p.lse && tid < 8) p.lse[static_cast<size_t>(b) * kH + h0 + tid] = lse_s[tid];
}

// ------------------------------------------------------------------------------------
// CUDA-core kernel (any dtype, D <= 1024): one CTA per (head, sequence), online softmax
// over 256-key chunks.

constexpr int kSimtChunk = 256;

__global__ void __launch_bounds__(256) mqa_simt_kernel(const MqaLaunch p, float scale_log2) {
  pdl_wait();
  pdl_launch_dependents();
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
  for (int d = tid; d < D; d += 256) {
    const size_t off = (static_cast<size_t>(b) * p.H + h) * D + d;
    if (p.out_dt == DSV4_F32) static_cast<float *>(p.out)[off] = ob[d];
    else static_cast<uint16_t *>(p.out)[off] = float_to_bf16_bits(ob[d]);
  }
  if (p.lse && tid == 0)
    p.lse[static_cast<size_t>(b) * p.H + h] = l_run > 0.f ? (m_run + log2f(l_run)) * kLn2 : -INFINITY;
}

int tc_grid() { return sm_count(); }

float softmax_scale_log2(const MqaLaunch &p) {
  const float s = p.softmax_scale > 0.f ? p.softmax_scale : 1.0f / sqrtf(static_cast<float>(p.D));
  return s * kLog2e;
}

}  // namespace

bool mqa_uses_tensor_cores(const MqaLaunch &p) {
  return (p.kv_dt == DSV4_BF16 || p.kv_dt == DSV4_FP8E4M3) && p.D == kD && p.H == kH && p.q_dt == DSV4_BF16 &&
         p.rope_dims % 8 == 0 && p.B <= 1024;
}

size_t mqa_workspace_bytes(const MqaLaunch &p) {
  if (!mqa_uses_tensor_cores(p)) return 0;
  const size_t slots = static_cast<size_t>(p.B) + tc_grid();
  return align_up(slots * kH * kD * sizeof(float), 256) + align_up(slots * kH * 2 * sizeof(float), 256) +
         align_up(static_cast<size_t>(p.B) * kH * kD * sizeof(uint16_t), 256) +
         align_up(static_cast<size_t>(p.B) * kH * sizeof(float), 256);
}

cudaError_t launch_mqa(const MqaLaunch &p0, void *ws, cudaStream_t st) {
  MqaLaunch p = p0;
  p.rope_theta1 = rope_theta1(p.rope_base, p.rope_dims);
  if (mqa_uses_tensor_cores(p)) {
    MqaTcParams P;
    P.a = p;
    P.scale_log2 = softmax_scale_log2(p);
    const size_t slots = static_cast<size_t>(p.B) + tc_grid();
    char *w = static_cast<char *>(ws);
    P.part_o = reinterpret_cast<float *>(w);
    w += align_up(slots * kH * kD * sizeof(float), 256);
    P.part_ml = reinterpret_cast<float *>(w);
    w += align_up(slots * kH * 2 * sizeof(float), 256);
    P.qp = reinterpret_cast<uint16_t *>(w);
    w += align_up(static_cast<size_t>(p.B) * kH * kD * sizeof(uint16_t), 256);
    P.qinv = reinterpret_cast<float *>(w);
    cudaError_t e = launch_pdl(mqa_query_kernel, dim3(p.B), dim3(256), 0, st, 1, P);
    if (e != cudaSuccess) return e;
    const size_t smem = sizeof(MqaSmem) + 1024 + (static_cast<size_t>(p.B) + 1 + kThreads) * sizeof(long long);
    e = cudaFuncSetAttribute(mqa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = launch_pdl(mqa_tc_kernel, dim3(tc_grid()), dim3(kThreads), smem, st, 1, P);
    if (e != cudaSuccess) return e;
    const size_t msmem = static_cast<size_t>(tc_grid()) * 16 * sizeof(float) +
                         static_cast<size_t>((tc_grid() + 1) & ~1) * sizeof(int) +
                         (static_cast<size_t>(p.B) + 1 + 256) * sizeof(long long);
    e = cudaFuncSetAttribute(mqa_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(mqa_merge_kernel, dim3(p.B, kH / 8), dim3(256), msmem, st, 1, P, tc_grid());
  }
  const size_t smem = (2 * static_cast<size_t>(p.D) + 2 * kSimtChunk + 32) * sizeof(float) +
                      kSimtChunk * sizeof(void *) + 16;
  cudaError_t e = cudaFuncSetAttribute(mqa_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(mqa_simt_kernel, dim3(p.H, p.B), dim3(256), smem, st, 1, p, softmax_scale_log2(p));
}

}  // namespace dsv4
