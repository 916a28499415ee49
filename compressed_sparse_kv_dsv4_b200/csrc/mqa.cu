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
// every thread of the CTA (contiguous slices of sequences, then a scan of the slices).
// red: blockDim.x scratch values.
__device__ void chunk_prefix(const MqaLaunch &p, long long *prefix, long long *red, bool report_it) {
  const int nt = blockDim.x, t = threadIdx.x;
  const int lo = static_cast<int>((static_cast<long long>(p.B) * t) / nt);
  const int hi = static_cast<int>((static_cast<long long>(p.B) * (t + 1)) / nt);
  long long mine = 0;
  for (int b = lo; b < hi; ++b) {
    const KeyList L = key_list(p, b, report_it);
    const long long c = (L.nw + L.nsel + 63) / 64;
    prefix[b] = c;
    mine += c;
  }
  red[t] = mine;
  __syncthreads();
  if (t == 0) {
    long long acc = 0;
    for (int i = 0; i < nt; ++i) {
      const long long v = red[i];
      red[i] = acc;
      acc += v;
    }
    prefix[p.B] = acc;
  }
  __syncthreads();
  long long acc = red[t];
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

constexpr int kH = 64, kD = 512, kCh = 64, kThreads = 256;
constexpr int kAtom = kCh * 128;  // one 64-dim column block of a 64-row tile: 8 KB
constexpr int kMetaChunks = 8;

struct alignas(1024) MqaSmem {
  uint8_t q[kD / 64][kH * 128];      // 64 KB, K-major SW128, 8 atoms of 64 dims
  uint8_t k[2][kD / 64][kCh * 128];  // 2 x 64 KB
  uint8_t p[kH * 128];               // 8 KB: P[64 heads][64 keys], K-major SW128
  const uint8_t *rowp[2][kCh];
  float rscale[2][kCh];              // row scale of each key (0: no key)
  // key metadata of up to kMetaChunks consecutive chunks, resolved together so the
  // idx -> block table -> scale load chain is paid once per batch, not once per chunk
  const uint8_t *mrow[kMetaChunks * kCh];
  float mscale[kMetaChunks * kCh];
  KeyList mkl[kMetaChunks];
  int mb[kMetaChunks];
  long long mlc[kMetaChunks];
  long long meta_first;
  int meta_n;
  float cs[kD / 2], sn[kD / 2];
  float qinv[kH];                    // 2^-e of the per-head query scale (fp16 operands)
  float smax[2][2];                  // per-warp max row scale of a chunk being gathered
  int ec[2];                         // chunk exponent: K rows hold code * scale * 2^-ec
  unsigned qmax[kH];
  uint64_t bar_s, bar_o;
  uint32_t tmem_base;
  int abort_flag;
};

struct MqaTcParams {
  MqaLaunch a;
  float scale_log2;
  float *part_o;   // [B + G][H][D]
  float *part_ml;  // [B + G][H][2]
};

// Operands of the two MMAs. fp8 caches: fp16 (e4m3 -> fp16 is exact, and fp16 keeps 11
// significand bits of the rotated query and of P); bf16 caches: bf16.
__device__ __forceinline__ bool fp16_operands(const MqaLaunch &p) { return p.kv_dt == DSV4_FP8E4M3; }

__device__ __forceinline__ uint32_t pack_f16x2(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t *>(&h);
}

// Resolve the row address and scale of every key of chunks [g0, g0 + n) (n <= kMetaChunks).
__device__ void resolve_meta(const MqaTcParams &P, MqaSmem &S, const long long *prefix, long long g0, long long c1) {
  const MqaLaunch &p = P.a;
  const int tid = threadIdx.x;
  const int n = static_cast<int>(c1 - g0 < kMetaChunks ? c1 - g0 : kMetaChunks);
  if (tid < n) {
    const int b = find_seq(prefix, p.B, g0 + tid);
    S.mb[tid] = b;
    S.mlc[tid] = g0 + tid - prefix[b];
    S.mkl[tid] = key_list(p, b, false);
  }
  __syncthreads();
  // the cached range changes only after every thread has passed the barrier above, that
  // is, after every thread has taken its decision to resolve from the old range
  if (tid == 0) {
    S.meta_first = g0;
    S.meta_n = n;
  }
  for (int i = tid; i < n * kCh; i += kThreads) {
    const int c = i / kCh;
    const KeyList &L = S.mkl[c];
    const long long t = S.mlc[c] * kCh + (i % kCh);
    float sc = 0.f;
    const uint8_t *rp = t < L.nw + L.nsel ? key_row(p, S.mb[c], L, t, &sc) : nullptr;
    S.mrow[i] = rp;
    S.mscale[i] = rp ? sc : 0.f;
  }
  __syncthreads();
}

// Gather one 64-key chunk into a swizzled K-major tile. For fp8 rows the row scale is
// folded in: tile row j = code_j * (scale_j * 2^-ec) in fp16, with ec the exponent of the
// chunk's largest row scale, so every tile value stays within +-448.
__device__ void gather_chunk(const MqaTcParams &P, MqaSmem &S, const long long *prefix, long long g, long long c1,
                             int kb) {
  const MqaLaunch &p = P.a;
  const int tid = threadIdx.x;
  if (g < S.meta_first || g >= S.meta_first + S.meta_n) resolve_meta(P, S, prefix, g, c1);
  if (tid < kCh) {
    const int i = static_cast<int>(g - S.meta_first) * kCh + tid;
    const uint8_t *rp = S.mrow[i];
    const float sc = S.mscale[i];
    S.rowp[kb][tid] = rp;
    S.rscale[kb][tid] = sc;
    const float wm = warp_max(sc);
    if ((tid & 31) == 0) S.smax[kb][tid >> 5] = wm;
  }
  __syncthreads();
  uint8_t *kt = &S.k[kb][0][0];
  if (p.kv_dt == DSV4_FP8E4M3) {
    int ec = 0;
    frexpf(fmaxf(S.smax[kb][0], S.smax[kb][1]), &ec);  // max scale = f * 2^ec, f in [0.5, 1)
    if (tid == 0) S.ec[kb] = ec;
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sid = i * kThreads + tid, row = sid >> 5, seg = sid & 31;
      const uint8_t *rp = S.rowp[kb][row];
      v[i] = rp ? __ldg(reinterpret_cast<const uint4 *>(rp + seg * 16)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int sid = i * kThreads + tid, row = sid >> 5, seg = sid & 31;
      const __half2 sc2 = __float2half2_rn(ldexpf(S.rscale[kb][row], -ec));
      const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
      uint32_t o[8];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        __half2_raw a = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[u] & 0xFFFF), __NV_E4M3);
        __half2_raw c = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(w[u] >> 16), __NV_E4M3);
        __half2 ha = __hmul2(*reinterpret_cast<__half2 *>(&a), sc2);
        __half2 hc = __hmul2(*reinterpret_cast<__half2 *>(&c), sc2);
        o[2 * u] = *reinterpret_cast<uint32_t *>(&ha);
        o[2 * u + 1] = *reinterpret_cast<uint32_t *>(&hc);
      }
      const int atom = seg >> 2, c0 = (seg & 3) * 2;
      uint8_t *base = kt + atom * kAtom;
      *reinterpret_cast<uint4 *>(base + sw128_offset(row, c0)) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4 *>(base + sw128_offset(row, c0 + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
    }
  } else {  // bf16 rows: straight 16-byte copies into the swizzled tile
    if (tid == 0) S.ec[kb] = 0;
    uint4 v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int sid = i * kThreads + tid, row = sid >> 6, seg = sid & 63;
      const uint8_t *rp = S.rowp[kb][row];
      v[i] = rp ? __ldg(reinterpret_cast<const uint4 *>(rp + seg * 16)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int sid = i * kThreads + tid, row = sid >> 6, seg = sid & 63;
      *reinterpret_cast<uint4 *>(kt + (seg >> 3) * kAtom + sw128_offset(row, seg & 7)) = v[i];
    }
  }
}

// rotated query of sequence b, K-major swizzled: bf16, or fp16 scaled per head by a power
// of two (qinv[h] undoes it in the logits) so that |q| < 2^14 whatever the input range.
// A bf16 query is loaded once, all 16 segments of a thread up front.
__device__ void load_query(const MqaTcParams &P, MqaSmem &S, int b, int64_t pos) {
  const MqaLaunch &p = P.a;
  const int tid = threadIdx.x;
  const int half = p.rope_dims / 2;
  const bool f16 = fp16_operands(p);
  const bool raw_bf16 = p.q_dt == DSV4_BF16;
  uint4 raw[16];
  if (raw_bf16) {
    const uint16_t *q = static_cast<const uint16_t *>(p.q) + static_cast<size_t>(b) * kH * kD;
#pragma unroll
    for (int i = 0; i < 16; ++i) raw[i] = __ldg(reinterpret_cast<const uint4 *>(q) + i * kThreads + tid);
  }
  for (int i = tid; i < half; i += kThreads) rope_cos_sin(pos, i, p.rope_dims, p.rope_base, &S.cs[i], &S.sn[i]);
  if (tid < kH) S.qmax[tid] = 0u;
  __syncthreads();
  const int rope0 = kD - p.rope_dims;
  for (int pass = f16 ? 0 : 1; pass < 2; ++pass) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int sid = i * kThreads + tid, h = sid >> 6, seg = sid & 63;
      float x[8];
      if (raw_bf16) {
        const uint32_t w[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          x[2 * k] = __uint_as_float(w[k] << 16);
          x[2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
        }
      } else {
        load_row_f<8>(p.q, p.q_dt, (static_cast<size_t>(b) * kH + h) * kD + seg * 8, x);
      }
      const int d0 = seg * 8;
      if (d0 >= rope0) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int pi = (d0 + 2 * u - rope0) >> 1;
          const float c = S.cs[pi], s = S.sn[pi];
          const float x0 = x[2 * u], x1 = x[2 * u + 1];
          x[2 * u] = x0 * c - x1 * s;
          x[2 * u + 1] = x0 * s + x1 * c;
        }
      }
      if (pass == 0) {  // per-head max |q| (32 lanes of a warp cover half a head)
        float am = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) am = fmaxf(am, fabsf(x[u]));
        am = warp_max(am);
        if ((tid & 31) == 0) atomicMax(&S.qmax[h], __float_as_uint(am));
        continue;
      }
      uint4 o;
      if (f16) {
        const float qs = 1.0f / S.qinv[h];
        o = make_uint4(pack_f16x2(x[0] * qs, x[1] * qs), pack_f16x2(x[2] * qs, x[3] * qs),
                       pack_f16x2(x[4] * qs, x[5] * qs), pack_f16x2(x[6] * qs, x[7] * qs));
      } else {
        o = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                       pack_bf16x2(x[6], x[7]));
      }
      *reinterpret_cast<uint4 *>(&S.q[seg >> 3][0] + sw128_offset(h, seg & 7)) = o;
    }
    if (pass == 0) {
      __syncthreads();
      if (tid < kH) {
        int e = 0;
        const float am = __uint_as_float(S.qmax[tid]);
        if (am > 0.f) frexpf(am, &e);                         // am < 2^e
        S.qinv[tid] = am > 0.f ? ldexpf(1.0f, e - 14) : 1.0f;  // scaled |q| < 2^14
      }
      __syncthreads();
    }
  }
  if (!f16 && tid < kH) S.qinv[tid] = 1.0f;
}

__global__ void __launch_bounds__(kThreads, 1) mqa_tc_kernel(const __grid_constant__ MqaTcParams P) {
  extern __shared__ uint8_t smem_raw[];
  MqaSmem &S = *reinterpret_cast<MqaSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const MqaLaunch &p = P.a;
  long long *prefix = reinterpret_cast<long long *>(&S + 1);  // [B + 1] chunks before sequence b
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (tid == 0) {
    mbar_init(&S.bar_s, 1);
    mbar_init(&S.bar_o, 1);
    S.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&S.tmem_base, 512);
    tmem_relinquish();
  }
  chunk_prefix(p, prefix, prefix + p.B + 1, blockIdx.x == 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const long long T = prefix[p.B], G = gridDim.x;
  const long long c0 = (T * blockIdx.x) / G, c1 = (T * (blockIdx.x + 1)) / G;

  const bool f16 = fp16_operands(p);
  const bool smax_thread = warp < 4 && lane >= 16;  // owns S/O row (head) 16*warp + lane - 16
  const int quad = warp & 3;
  const int head = quad * 16 + (lane & 15);
  // Online softmax in log2 units. With z_j = x_j + ec (x_j the logit of key j), the
  // accumulators hold O = sum_j 2^(z_j - R) * Krow_j and l = sum_j 2^(z_j - R) * 2^-ec, both
  // from the same rounded P, in units of 2^R; R is raised lazily (only when a chunk's max z
  // exceeds it by more than 8), so P stays <= 2^8 and O is rescaled rarely.
  float R = -INFINITY, l_run = 0.f;
  int cur_b = -1;
  bool first_in_seg = true;
  KeyList L{};
  const uint32_t idesc1 = f16 ? idesc_f16(kH, kCh, 0, 0) : idesc_bf16(kH, kCh, 0, 0);
  const uint32_t idesc2 = f16 ? idesc_f16(kH, 256, 0, 1) : idesc_bf16(kH, 256, 0, 1);
  const uint32_t s_tmem = tmem + (16u << 16);  // S accumulator: lanes 16..31 of each quadrant

  if (tid == 0) {
    S.meta_first = 0;
    S.meta_n = 0;
  }
  __syncthreads();
  if (c0 < c1) gather_chunk(P, S, prefix, c0, c1, 0);
  for (long long g = c0; g < c1; ++g) {
    const long long it = g - c0;
    const int kb = static_cast<int>(it & 1);
    const int b = find_seq(prefix, p.B, g);
    if (b != cur_b) {
      cur_b = b;
      first_in_seg = true;
      R = -INFINITY;
      l_run = 0.f;
      L = key_list(p, b, false);
      load_query(P, S, b, L.pos);
    }
    fence_proxy_async_smem();
    __syncthreads();
    const int ec = S.ec[kb];
    if (tid == 0) {
      tc_fence_after();
      const uint32_t qa = smem_u32(&S.q[0][0]), ka = smem_u32(&S.k[kb][0][0]);
#pragma unroll
      for (int kk = 0; kk < kD / 16; ++kk) {
        const uint32_t off = (kk >> 2) * (kH * 128) + (kk & 3) * 32;
        const uint32_t offk = (kk >> 2) * kAtom + (kk & 3) * 32;
        mma_bf16(s_tmem, sw128_desc(qa + off, 16, 1024), sw128_desc(ka + offk, 16, 1024), idesc1, kk > 0 ? 1u : 0u);
      }
      mma_commit(&S.bar_s);
    }
    // prefetch the next chunk while MMA1 runs (its buffer was released by MMA2 of it-1)
    if (g + 1 < c1) gather_chunk(P, S, prefix, g + 1, c1, kb ^ 1);
    bool ok = mbar_wait(&S.bar_s, static_cast<uint32_t>(it & 1), &S.abort_flag);
    ok = __all_sync(0xFFFFFFFFu, ok);
    tc_fence_after();
    float alpha = 1.f;
    bool need_rescale = false;
    if (warp < 4 && ok) {
      uint32_t r0[32], r1[32];
      tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16), r0);
      tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + 32, r1);
      tmem_ld_wait();
      if (smax_thread) {
        const float *rs = S.rscale[kb];
        // logit in log2 units of key j: acc * tau*log2(e) * qinv[h] * (fp8: 2^ec; bf16: 1)
        const float coef = P.scale_log2 * S.qinv[head] * ldexpf(1.0f, ec);
        const float fec = static_cast<float>(ec);
        float z[kCh];
        float mz = -INFINITY;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          z[j] = rs[j] != 0.f ? fmaf(__uint_as_float(r0[j]), coef, fec) : -INFINITY;
          z[j + 32] = rs[j + 32] != 0.f ? fmaf(__uint_as_float(r1[j]), coef, fec) : -INFINITY;
          mz = fmaxf(mz, fmaxf(z[j], z[j + 32]));
        }
        float Rn = R;
        if (mz > R + 8.f) Rn = mz;
        alpha = (Rn == R) ? 1.f : exp2f(R - Rn);  // R = -inf -> 0
        need_rescale = (Rn != R) && !first_in_seg;
        const float lsc = ldexpf(1.0f, -ec);
        float lsum = 0.f;
        uint32_t pk[kCh / 2];
#pragma unroll
        for (int j = 0; j < kCh; j += 2) {
          const float e0 = z[j] == -INFINITY ? 0.f : exp2f(z[j] - Rn);
          const float e1 = z[j + 1] == -INFINITY ? 0.f : exp2f(z[j + 1] - Rn);
          float r0f, r1f;
          if (f16) {
            __half2 h = __floats2half2_rn(e0, e1);
            pk[j / 2] = *reinterpret_cast<uint32_t *>(&h);
            const float2 back = __half22float2(h);
            r0f = back.x;
            r1f = back.y;
          } else {
            pk[j / 2] = pack_bf16x2(e0, e1);
            r0f = __uint_as_float(pk[j / 2] << 16);
            r1f = __uint_as_float(pk[j / 2] & 0xFFFF0000u);
          }
          lsum += r0f + r1f;  // the denominator uses the rounded P, like the numerator
        }
        l_run = l_run * alpha + lsum * lsc;
        R = Rn;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4 *>(S.p + sw128_offset(head, c)) =
              make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      }
      // O rows (lanes 0..15) take their head's rescale factor from lane + 16
      const float alpha_o = __shfl_sync(0xFFFFFFFFu, alpha, (lane & 15) + 16);
      const bool any = __any_sync(0xFFFFFFFFu, need_rescale);
      if (any) {
        for (int col = 0; col < kD; col += 32) {
          uint32_t r[32];
          const uint32_t addr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + col;
          tmem_ld32(addr, r);
          tmem_ld_wait();
          if (lane < 16) {
#pragma unroll
            for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha_o);
          }
          tmem_st32(addr, r);
        }
        tmem_st_wait();
      }
    }
    if (!ok && lane == 0) S.abort_flag = 1;
    tc_fence_before();
    fence_proxy_async_smem();
    __syncthreads();
    if (S.abort_flag) break;
    if (tid == 0) {
      tc_fence_after();
      const uint32_t pa = smem_u32(S.p), ka = smem_u32(&S.k[kb][0][0]);
#pragma unroll
      for (int nh = 0; nh < 2; ++nh)
#pragma unroll
        for (int ks = 0; ks < kCh / 16; ++ks)
          mma_bf16(tmem + nh * 256, sw128_desc(pa + ks * 32, 16, 1024),
                   sw128_desc(ka + nh * 4 * kAtom + ks * 2048, kAtom, 1024), idesc2,
                   (!first_in_seg || ks > 0) ? 1u : 0u);
      mma_commit(&S.bar_o);
    }
    ok = mbar_wait(&S.bar_o, static_cast<uint32_t>(it & 1), &S.abort_flag);
    ok = __all_sync(0xFFFFFFFFu, ok);
    tc_fence_after();
    first_in_seg = false;
    const bool seg_end = (g + 1 == c1) || (find_seq(prefix, p.B, g + 1) != b);
    if (seg_end && ok) {
      const size_t slot = static_cast<size_t>(b) + blockIdx.x;
      if (smax_thread) {
        float *ml = P.part_ml + (slot * kH + head) * 2;
        ml[0] = R;
        ml[1] = l_run;
      }
      // all 8 warps read O: warps 0-3 columns 0..255, warps 4-7 columns 256..511
      const int colbase = (warp >> 2) * 256;
      float *po = P.part_o + (slot * kH + head) * kD;
      for (int col = colbase; col < colbase + 256; col += 32) {
        uint32_t r[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(quad * 32) << 16) + col, r);
        tmem_ld_wait();
        if (lane < 16) {
#pragma unroll
          for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(po + col + i) = make_float4(
                __uint_as_float(r[i]), __uint_as_float(r[i + 1]), __uint_as_float(r[i + 2]), __uint_as_float(r[i + 3]));
        }
      }
      tc_fence_before();
    }
    if (!ok && lane == 0) S.abort_flag = 1;
    __syncthreads();
    if (S.abort_flag) break;
  }

  if (tid == 0 && S.abort_flag) report(p.d_status, DSV4_DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the partials of every sequence, inverse RoPE, store. grid (B, H / 8), 256 threads.
__global__ void __launch_bounds__(256) mqa_merge_kernel(const MqaTcParams P, int grid_ctas) {
  const MqaLaunch &p = P.a;
  __shared__ int np_s;  // partials of this sequence
  __shared__ float cs[kD / 2], sn[kD / 2];
  extern __shared__ __align__(16) uint8_t dyn[];
  float *wgt = reinterpret_cast<float *>(dyn);  // [grid_ctas][8]: weight of each partial, per head
  int *cta = reinterpret_cast<int *>(wgt + static_cast<size_t>(grid_ctas) * 8);  // [grid_ctas]
  long long *prefix = reinterpret_cast<long long *>(cta + ((grid_ctas + 1) & ~1));  // [B + 1]
  long long *red = prefix + p.B + 1;                                             // [blockDim]
  __shared__ float inv_l[8], lse_s[8];
  const int b = blockIdx.x, h0 = blockIdx.y * 8, tid = threadIdx.x;
  chunk_prefix(p, prefix, red, false);
  if (tid == 0) {
    // the CTAs of the main kernel whose (non-empty) chunk range meets this sequence; with
    // fewer chunks than CTAs some ranges are empty and those CTAs wrote no partial
    const long long acc = prefix[p.B], mine = prefix[b], cnt = prefix[b + 1] - prefix[b];
    int n = 0;
    for (int c = 0; c < grid_ctas && cnt > 0; ++c) {
      const long long a0 = (acc * c) / grid_ctas, a1 = (acc * (c + 1)) / grid_ctas;
      if (a0 < mine + cnt && a1 > mine && a1 > a0) cta[n++] = c;
    }
    np_s = n;
  }
  const KeyList L = key_list(p, b, false);
  const int half = p.rope_dims / 2;
  for (int i = tid; i < half; i += 256) rope_cos_sin(L.pos, i, p.rope_dims, p.rope_base, &cs[i], &sn[i]);
  __syncthreads();
  const int np = np_s;
  if (tid < 8) {
    const int h = h0 + tid;
    float M = -INFINITY;
    for (int i = 0; i < np; ++i) {
      const size_t slot = static_cast<size_t>(b) + cta[i];
      M = fmaxf(M, P.part_ml[(slot * kH + h) * 2]);
    }
    float Ls = 0.f;
    for (int i = 0; i < np; ++i) {
      const size_t slot = static_cast<size_t>(b) + cta[i];
      const float mi = P.part_ml[(slot * kH + h) * 2], li = P.part_ml[(slot * kH + h) * 2 + 1];
      const float w = (mi == -INFINITY) ? 0.f : exp2f(mi - M);
      wgt[i * 8 + tid] = w;
      Ls += w * li;
    }
    inv_l[tid] = Ls > 0.f ? 1.f / Ls : 0.f;
    lse_s[tid] = Ls > 0.f ? (M + log2f(Ls)) * kLn2 : -INFINITY;
  }
  __syncthreads();
  const int rope0 = kD - p.rope_dims;
  for (int t = tid; t < 8 * (kD / 2); t += 256) {
    const int hh = t / (kD / 2), pr = t % (kD / 2), h = h0 + hh;
    float o0 = 0.f, o1 = 0.f;
    for (int i = 0; i < np; ++i) {
      const size_t slot = static_cast<size_t>(b) + cta[i];
      const float2 v = *reinterpret_cast<const float2 *>(P.part_o + (slot * kH + h) * kD + 2 * pr);
      o0 = fmaf(wgt[i * 8 + hh], v.x, o0);
      o1 = fmaf(wgt[i * 8 + hh], v.y, o1);
    }
    o0 *= inv_l[hh];
    o1 *= inv_l[hh];
    const int d = 2 * pr;
    if (d >= rope0) {  // rotate by -pos
      const int pi = (d - rope0) >> 1;
      const float c = cs[pi], s = sn[pi];
      const float y0 = o0 * c + o1 * s, y1 = -o0 * s + o1 * c;
      o0 = y0;
      o1 = y1;
    }
    const size_t off = (static_cast<size_t>(b) * kH + h) * kD + d;
    if (p.out_dt == DSV4_F32) {
      *reinterpret_cast<float2 *>(static_cast<float *>(p.out) + off) = make_float2(o0, o1);
    } else {
      *reinterpret_cast<uint32_t *>(static_cast<uint16_t *>(p.out) + off) = pack_bf16x2(o0, o1);
    }
  }
  if (p.lse && tid < 8) p.lse[static_cast<size_t>(b) * kH + h0 + tid] = lse_s[tid];
}

// ------------------------------------------------------------------------------------
// CUDA-core kernel (any dtype, D <= 1024): one CTA per (head, sequence), online softmax
// over 256-key chunks.

constexpr int kSimtChunk = 256;

__global__ void __launch_bounds__(256) mqa_simt_kernel(const MqaLaunch p, float scale_log2) {
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
    rope_cos_sin(L.pos, i, p.rope_dims, p.rope_base, &c, &s);
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
    rope_cos_sin(L.pos, i, p.rope_dims, p.rope_base, &c, &s);
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
  return (p.kv_dt == DSV4_BF16 || p.kv_dt == DSV4_FP8E4M3) && p.D == kD && p.H == kH &&
         (p.q_dt == DSV4_BF16 || p.q_dt == DSV4_F32) && p.rope_dims % 8 == 0 && p.B <= 1024;
}

size_t mqa_workspace_bytes(const MqaLaunch &p) {
  if (!mqa_uses_tensor_cores(p)) return 0;
  const size_t slots = static_cast<size_t>(p.B) + tc_grid();
  return align_up(slots * kH * kD * sizeof(float), 256) + align_up(slots * kH * 2 * sizeof(float), 256);
}

cudaError_t launch_mqa(const MqaLaunch &p, void *ws, cudaStream_t st) {
  if (mqa_uses_tensor_cores(p)) {
    MqaTcParams P;
    P.a = p;
    P.scale_log2 = softmax_scale_log2(p);
    const size_t slots = static_cast<size_t>(p.B) + tc_grid();
    P.part_o = static_cast<float *>(ws);
    P.part_ml = reinterpret_cast<float *>(static_cast<char *>(ws) + align_up(slots * kH * kD * sizeof(float), 256));
    const size_t smem = sizeof(MqaSmem) + 1024 + (static_cast<size_t>(p.B) + 1 + kThreads) * sizeof(long long);
    cudaError_t e = cudaFuncSetAttribute(mqa_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    mqa_tc_kernel<<<tc_grid(), kThreads, smem, st>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t msmem = static_cast<size_t>(tc_grid()) * 8 * sizeof(float) +
                         static_cast<size_t>((tc_grid() + 1) & ~1) * sizeof(int) +
                         (static_cast<size_t>(p.B) + 1 + 256) * sizeof(long long);
    e = cudaFuncSetAttribute(mqa_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)msmem);
    if (e != cudaSuccess) return e;
    mqa_merge_kernel<<<dim3(p.B, kH / 8), 256, msmem, st>>>(P, tc_grid());
    return cudaGetLastError();
  }
  const size_t smem = (2 * static_cast<size_t>(p.D) + 2 * kSimtChunk + 32) * sizeof(float) +
                      kSimtChunk * sizeof(void *) + 16;
  cudaError_t e = cudaFuncSetAttribute(mqa_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  mqa_simt_kernel<<<dim3(p.H, p.B), 256, smem, st>>>(p, softmax_scale_log2(p));
  return cudaGetLastError();
}

}  // namespace dsv4
