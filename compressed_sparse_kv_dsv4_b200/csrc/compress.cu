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
// The work is bandwidth-bound: a row of D channels is covered by D/8 threads (8 channels, one
// 16-byte bf16 load per token each); a thread keeps several tokens' loads in flight and pools
// its channels in float32 registers (a softmax in log2 units). Long blocks are split into token
// slices merged in shared memory. Norm, rotation, rounding and store follow in registers.
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

// RMSNorm(e) * gamma, RoPE at `rope_pos`, round into `dt`, store to `row` (+ *scale_out).
// e: shared float[D]; red: shared float[32]. Every thread of the CTA calls this.
__device__ void finish_and_store(float *e, int D, const float *gamma, float eps, int64_t rope_pos, int rope_dims,
                                 double rope_theta1, dsv4_dtype dt, void *row, float *scale_out, float *red) {
  const int tid = threadIdx.x;
  float ss = 0.f;
  for (int c = tid; c < D; c += static_cast<int>(blockDim.x)) ss += e[c] * e[c];
  ss = block_sum(ss, red);
  const float rs = 1.0f / sqrtf(ss / static_cast<float>(D) + eps);
  __syncthreads();
  for (int c = tid; c < D; c += static_cast<int>(blockDim.x)) e[c] = e[c] * rs * gamma[c];
  __syncthreads();
  const int half = rope_dims / 2;
  for (int i = tid; i < half; i += static_cast<int>(blockDim.x)) {
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
    for (int c = tid; c < D; c += static_cast<int>(blockDim.x)) o[c] = e[c];
  } else if (dt == DSV4_BF16) {
    uint16_t *o = static_cast<uint16_t *>(row);
    for (int c = tid; c < D; c += static_cast<int>(blockDim.x)) o[c] = float_to_bf16_bits(e[c]);
  } else {
    float am = 0.f;
    for (int c = tid; c < D; c += static_cast<int>(blockDim.x)) am = fmaxf(am, fabsf(e[c]));
    am = block_max(am, red);
    const float scale = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
    const float inv = am > 0.f ? __fdiv_rn(448.0f, am) : 1.0f;
    uint8_t *o = static_cast<uint8_t *>(row);
    for (int c2 = tid; c2 < D / 2; c2 += static_cast<int>(blockDim.x)) {
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
  return static_cast<char *>(pages) + dtype_bytes(dt, r * D);
}

// items of sequence s: one per completed block, at least one (the state-tail write)
__device__ __forceinline__ int64_t compress_items(const SeqRange &r, int m) {
  const int64_t c = r.p1 / m - r.p0 / m;
  return c > 1 ? c : 1;
}

// ---- prefill: a row of D channels is covered by a "row group" of R = D / 8 threads, 8
// consecutive channels each (one 16-byte load per bf16 token row). A CTA holds NG = kThreads / R
// row groups. Each completed block is pooled by S row groups, each over a contiguous slice of
// m / S tokens (S = 1 for short blocks: the group holds the whole block in registers), so a
// CTA takes NG / S blocks at once. Every thread keeps several tokens' loads in flight.

constexpr int kTokUnroll = 4;  // tokens whose loads one thread issues together

struct PrefillShape {
  int R, NG, S, BPC;  // threads per row, row groups per CTA, groups per block, blocks per CTA
};

__host__ __device__ inline PrefillShape prefill_shape(int D, int m, int threads = kThreads) {
  PrefillShape sh;
  sh.R = D / 8;
  sh.NG = threads / sh.R > 0 ? threads / sh.R : 1;
  int s = m / 8 > 1 ? m / 8 : 1;
  sh.S = s < sh.NG ? s : sh.NG;
  sh.BPC = sh.NG / sh.S;
  return sh;
}

// The 8 channels [8 cg, 8 cg + 8) of token t's kv (state ring or input row).
__device__ __forceinline__ void load_kv8(const TokenSource &src, int64_t t, int cg, float (&v)[8]) {
  const int D = src.D, G = src.G;
  if (t < src.p0) {
    const float *row = src.state + static_cast<size_t>(t % src.m) * (D + G);
    if (G == D) {  // rows of 2D floats: 16-byte aligned
      load_row_f<8>(row, DSV4_F32, static_cast<size_t>(cg) * 8, v);
    } else {  // rows of D + 1 floats: scalar loads
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = row[cg * 8 + i];
    }
  } else {
    const size_t r = static_cast<size_t>(src.row0 + (t - src.p0));
    load_row_f<8>(src.kv, src.kv_dt, r * D + static_cast<size_t>(cg) * 8, v);
  }
}

// The gates of those channels (the token's one gate, broadcast, when G = 1).
__device__ __forceinline__ void load_gate8(const TokenSource &src, int64_t t, int cg, float (&g)[8]) {
  const int D = src.D, G = src.G;
  if (t < src.p0) {
    const float *row = src.state + static_cast<size_t>(t % src.m) * (D + G);
    if (G == D) {
      load_row_f<8>(row + D, DSV4_F32, static_cast<size_t>(cg) * 8, g);
    } else {
      const float g0 = row[D];
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = g0;
    }
  } else {
    const size_t r = static_cast<size_t>(src.row0 + (t - src.p0));
    if (G == D) {
      load_row_f<8>(src.gate, src.kv_dt, r * G + static_cast<size_t>(cg) * 8, g);
    } else {
      const float g0 = load_one_f(src.gate, src.kv_dt, r * G);
#pragma unroll
      for (int i = 0; i < 8; ++i) g[i] = g0;
    }
  }
}

__device__ __forceinline__ void load_token8(const TokenSource &src, int64_t t, int cg, float (&v)[8], float (&g)[8]) {
  load_kv8(src, t, cg, v);
  load_gate8(src, t, cg, g);
}

// Ring slot of position t (a new token of a block completed in this call) may be written by
// the group that pooled its block: the slot is not one of those the sequence's first block
// reads from earlier calls (positions [first block start, p0), slots below p0 % m), or t is in
// that first block itself (its group read those slots before writing).
__device__ __forceinline__ bool ring_slot_safe(const SeqRange &r, int m, int64_t t) {
  const int64_t off = r.p0 % m;
  return off == 0 || t / m == r.p0 / m || t % m >= off;
}

// kv (and gate) of one token, 8 channels [8 cg, 8 cg + 8), into its float32 ring row.
__device__ __forceinline__ void store_token8(float *row, int D, int G, int cg, const float (&v)[8], float g0,
                                             const float (&g)[8]) {
  if (G == D) {  // rows of 2D floats: 16-byte aligned
    float4 *o = reinterpret_cast<float4 *>(row + cg * 8);
    o[0] = make_float4(v[0], v[1], v[2], v[3]);
    o[1] = make_float4(v[4], v[5], v[6], v[7]);
    float4 *og = reinterpret_cast<float4 *>(row + D + cg * 8);
    og[0] = make_float4(g[0], g[1], g[2], g[3]);
    og[1] = make_float4(g[4], g[5], g[6], g[7]);
  } else {
#pragma unroll
    for (int c = 0; c < 8; ++c) row[cg * 8 + c] = v[c];
    if (cg == 0) row[D] = g0;
  }
}

// Sum (or max) of v over the thread's row group of R threads (a power of two). Every thread
// of the CTA calls it (it may synchronize the CTA); red holds kThreads / 32 floats.
__device__ __forceinline__ float group_reduce(float v, int R, float *red, bool is_max) {
  const int w = R < 32 ? R : 32;
  for (int o = w >> 1; o > 0; o >>= 1) {
    const float u = __shfl_xor_sync(0xFFFFFFFFu, v, o);
    v = is_max ? fmaxf(v, u) : v + u;
  }
  if (R <= 32) return v;
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  const int wpg = R >> 5, w0 = (static_cast<int>(threadIdx.x) >> 5) / wpg * wpg;
  float t = red[w0];
  for (int i = 1; i < wpg; ++i) t = is_max ? fmaxf(t, red[w0 + i]) : t + red[w0 + i];
  __syncthreads();
  return t;
}

// Up to kTokUnroll tokens (the first n_valid) of one channel folded into its running softmax
// pool, in log2 units: gl = gate * log2(e), weights 2^(gl - max). Every operation is rounded
// on its own (no contraction the compiler might choose differently from one call site to
// another), so the bytes a block stores do not depend on which path loaded its tokens.
__device__ __forceinline__ void pool_channel(const float (&v)[kTokUnroll], const float (&gl)[kTokUnroll], int n_valid,
                                             float &mx, float &l, float &acc) {
  float bm = mx;
#pragma unroll
  for (int k = 0; k < kTokUnroll; ++k)
    if (k < n_valid) bm = fmaxf(bm, gl[k]);
  const float a = ex2_approx(__fsub_rn(mx, bm));  // 0 while nothing was pooled (mx = -inf)
  float sa = __fmul_rn(acc, a), sw = __fmul_rn(l, a);
#pragma unroll
  for (int k = 0; k < kTokUnroll; ++k) {
    if (k < n_valid) {
      const float w = ex2_approx(__fsub_rn(gl[k], bm));
      sa = fmaf(w, v[k], sa);
      sw = __fadd_rn(sw, w);
    }
  }
  acc = sa;
  l = sw;
  mx = bm;
}

// value c (0..7) of 8 packed bf16
__device__ __forceinline__ float bf16_lane(const uint4 &r, int c) {
  const uint32_t w = c < 2 ? r.x : (c < 4 ? r.y : (c < 6 ? r.z : r.w));
  return __uint_as_float((c & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

// kv and gate (8 packed bf16 each, channels [8 cg, 8 cg + 8)) into a float32 ring row of 2D floats
__device__ __forceinline__ void store_token_bf16(float *row, int D, int cg, const uint4 &k, const uint4 &g) {
  float4 *o = reinterpret_cast<float4 *>(row + cg * 8);
  o[0] = make_float4(bf16_lane(k, 0), bf16_lane(k, 1), bf16_lane(k, 2), bf16_lane(k, 3));
  o[1] = make_float4(bf16_lane(k, 4), bf16_lane(k, 5), bf16_lane(k, 6), bf16_lane(k, 7));
  float4 *og = reinterpret_cast<float4 *>(row + D + cg * 8);
  og[0] = make_float4(bf16_lane(g, 0), bf16_lane(g, 1), bf16_lane(g, 2), bf16_lane(g, 3));
  og[1] = make_float4(bf16_lane(g, 4), bf16_lane(g, 5), bf16_lane(g, 6), bf16_lane(g, 7));
}

constexpr float kLog2eF = 1.4426950408889634f;

// What a compressor needs, whichever kernel runs it (the prefill, or a decode step's prologue).
struct CompressView {
  const void *kv, *gate;  // input rows [*][D], [*][G]
  dsv4_dtype kv_dt;
  const float *gamma;
  float eps;
  int rope_dims;
  double rope_theta1;
  float *state;  // [B][m][D + G]
  int m, D, G;
  void *pages;
  float *scales;
  const int32_t *block_table;
  int num_pages, max_blocks;
  dsv4_dtype cache_dt;
  uint32_t *d_status;
};

// One chunk: the CTA's row groups pool, finish and store up to BPC items (completed blocks),
// then store the state-ring tokens of the sequences whose first item is in the chunk. `map`
// gives an item's sequence, its index among the sequence's items and the sequence's range.
// The arithmetic of a block does not depend on where its tokens come from (input rows or the
// ring), so a prefill in one call and the same tokens fed one by one store the same bytes.
template <bool kEagerLoads, class Map>
__device__ void compress_chunk(const CompressView &p, const PrefillShape &sh, float *part, float *red, long long chunk,
                               long long total, const Map &map) {
  const int tid = threadIdx.x;
  const int grp = tid / sh.R, cg = tid % sh.R;  // row group, channel group (8 channels)
  const int li = grp / sh.S, sl = grp % sh.S;   // local block, slice of it
  const bool bf16_rows = p.kv_dt == DSV4_BF16 && p.G == p.D;
  const long long item = chunk * sh.BPC + li;
  int s = 0;
  int64_t i = 0;
  SeqRange r{0, 0, 0};
  bool has_block = false;
  if (item < total) {
    map.locate(item, &s, &i, &r);
    has_block = (r.p1 / p.m - r.p0 / p.m) > i;
  }
  float *st = p.state + static_cast<size_t>(s) * p.m * (p.D + p.G);
  const int64_t b = r.p0 / p.m + i;

  // pool this group's slice of the block, in batches of kTokUnroll tokens whose loads are in
  // flight together
  float mx[8], l[8], acc[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) { mx[c] = -INFINITY; l[c] = 0.f; acc[c] = 0.f; }
  if (has_block) {
    const int per = p.m / sh.S, u0 = sl * per, u1 = u0 + per;
    const int64_t tail_lo = r.p1 - p.m > r.p0 ? r.p1 - p.m : r.p0;  // the ring keeps positions >= tail_lo
    const bool from_input = b * p.m + u0 >= r.p0;                      // no token of the slice is in the ring
    for (int u = u0; u < u1; u += kTokUnroll) {
      const int nv = u1 - u < kTokUnroll ? u1 - u : kTokUnroll;
      if (bf16_rows && from_input) {
        // bf16 input rows: the raw 16-byte loads first, unpacked per channel
        const uint16_t *kv16 = static_cast<const uint16_t *>(p.kv), *g16 = static_cast<const uint16_t *>(p.gate);
        const size_t row = static_cast<size_t>(r.row0 + (b * p.m + u - r.p0));
        uint4 rk[kTokUnroll], rg[kTokUnroll];
#pragma unroll
        for (int k = 0; k < kTokUnroll; ++k) {
          if (k < nv) {
            rk[k] = __ldg(reinterpret_cast<const uint4 *>(kv16 + (row + k) * p.D) + cg);
            rg[k] = __ldg(reinterpret_cast<const uint4 *>(g16 + (row + k) * p.D) + cg);
          } else {
            rk[k] = make_uint4(0, 0, 0, 0);
            rg[k] = make_uint4(0, 0, 0, 0);
          }
        }
        // tokens the ring keeps go there from these registers, unless the slot is one the
        // sequence's first block still reads (written by its CTA, below)
#pragma unroll
        for (int k = 0; k < kTokUnroll; ++k) {
          const int64_t t = b * p.m + u + k;
          if (k < nv && t >= tail_lo && ring_slot_safe(r, p.m, t))
            store_token_bf16(st + static_cast<size_t>(t % p.m) * 2 * p.D, p.D, cg, rk[k], rg[k]);
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float vv[kTokUnroll], gg[kTokUnroll];
#pragma unroll
          for (int k = 0; k < kTokUnroll; ++k) {
            vv[k] = bf16_lane(rk[k], c);
            gg[k] = __fmul_rn(bf16_lane(rg[k], c), kLog2eF);
          }
          pool_channel(vv, gg, nv, mx[c], l[c], acc[c]);
        }
      } else {
        // other rows (float32 inputs, a scalar gate, or ring slots): the batch's gates first,
        // then its tokens' kv one by one, in the same order of operations as above
        const TokenSource src{st, p.kv, p.gate, p.kv_dt, r.p0, r.row0, p.m, p.D, p.G};
        float g[kTokUnroll][8];
#pragma unroll
        for (int k = 0; k < kTokUnroll; ++k) {
          if (k < nv) load_gate8(src, b * p.m + u + k, cg, g[k]);
          else {
#pragma unroll
            for (int c = 0; c < 8; ++c) g[k][c] = 0.f;
          }
        }
        // (kEagerLoads: every token's kv is loaded before the arithmetic, for the latency-bound
        // decode step; the arithmetic is the same either way)
        float ve[kEagerLoads ? kTokUnroll : 1][8];
        if (kEagerLoads) {
#pragma unroll
          for (int k = 0; k < (kEagerLoads ? kTokUnroll : 1); ++k)
            if (k < nv) load_kv8(src, b * p.m + u + k, cg, ve[k]);
        }
        float bm[8], sa[8], sw[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          bm[c] = mx[c];
#pragma unroll
          for (int k = 0; k < kTokUnroll; ++k)
            if (k < nv) bm[c] = fmaxf(bm[c], __fmul_rn(g[k][c], kLog2eF));
          const float a = ex2_approx(__fsub_rn(mx[c], bm[c]));
          sa[c] = __fmul_rn(acc[c], a);
          sw[c] = __fmul_rn(l[c], a);
        }
#pragma unroll
        for (int k = 0; k < kTokUnroll; ++k) {
          if (k < nv) {
            const int64_t t = b * p.m + u + k;
            float v[8];
            if (kEagerLoads) {
#pragma unroll
              for (int c = 0; c < 8; ++c) v[c] = ve[kEagerLoads ? k : 0][c];
            } else {
              load_kv8(src, t, cg, v);
            }
            if (t >= tail_lo && ring_slot_safe(r, p.m, t))
              store_token8(st + static_cast<size_t>(t % p.m) * (p.D + p.G), p.D, p.G, cg, v, g[k][0], g[k]);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float w = ex2_approx(__fsub_rn(__fmul_rn(g[k][c], kLog2eF), bm[c]));
              sa[c] = fmaf(w, v[c], sa[c]);
              sw[c] = __fadd_rn(sw[c], w);
            }
          }
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          acc[c] = sa[c];
          l[c] = sw[c];
          mx[c] = bm[c];
        }
      }
    }
  }
  // slices of one block merged in shared memory by its first group
  if (sh.S > 1) {
    float *mine = part + static_cast<size_t>(grp) * 3 * p.D + cg * 8;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      mine[c] = mx[c];
      mine[p.D + c] = l[c];
      mine[2 * p.D + c] = acc[c];
    }
    __syncthreads();
    if (sl == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        float M = -INFINITY;
        for (int k = 0; k < sh.S; ++k) M = fmaxf(M, part[static_cast<size_t>(grp + k) * 3 * p.D + cg * 8 + c]);
        float L = 0.f, A = 0.f;
        for (int k = 0; k < sh.S; ++k) {
          const float *q = part + static_cast<size_t>(grp + k) * 3 * p.D + cg * 8 + c;
          if (q[0] == -INFINITY) continue;
          const float w = ex2_approx(q[0] - M);
          L += w * q[p.D];
          A += w * q[2 * p.D];
        }
        l[c] = L;
        acc[c] = A;
      }
    }
    __syncthreads();  // part is rewritten by the next chunk
  }
  const bool owner = has_block && sl == 0;  // this group finishes the block
  float e[8];
#pragma unroll
  for (int c = 0; c < 8; ++c) e[c] = owner ? acc[c] / l[c] : 0.f;
  // RMSNorm over the row group, times gamma
  float ss = 0.f;
#pragma unroll
  for (int c = 0; c < 8; ++c) ss += e[c] * e[c];
  ss = group_reduce(ss, sh.R, red, false);
  const float rs = 1.0f / sqrtf(ss / static_cast<float>(p.D) + p.eps);
#pragma unroll
  for (int c = 0; c < 8; ++c) e[c] = e[c] * rs * __ldg(p.gamma + cg * 8 + c);
  // RoPE at the block position on the last rope_dims channels (pairs never straddle threads)
  const int rope0 = p.D - p.rope_dims;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int c0 = cg * 8 + 2 * j;
    if (owner && c0 >= rope0) {
      float cs, sn;
      rope_cos_sin(b * p.m, (c0 - rope0) >> 1, p.rope_theta1, &cs, &sn);
      const float x0 = e[2 * j], x1 = e[2 * j + 1];
      e[2 * j] = x0 * cs - x1 * sn;
      e[2 * j + 1] = x0 * sn + x1 * cs;
    }
  }
  float *sp = nullptr;
  void *row = nullptr;
  if (owner)
    row = cache_row(p.pages, p.scales, p.block_table, p.num_pages, p.max_blocks, p.m, p.D, p.cache_dt, s, b, &sp,
                    cg == 0 ? p.d_status : nullptr);
  if (p.cache_dt == DSV4_F32) {
    if (row) {
      float4 *o = reinterpret_cast<float4 *>(static_cast<float *>(row) + cg * 8);
      o[0] = make_float4(e[0], e[1], e[2], e[3]);
      o[1] = make_float4(e[4], e[5], e[6], e[7]);
    }
  } else if (p.cache_dt == DSV4_BF16) {
    if (row)
      *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(row) + cg * 8) =
          make_uint4(pack_bf16x2(e[0], e[1]), pack_bf16x2(e[2], e[3]), pack_bf16x2(e[4], e[5]),
                     pack_bf16x2(e[6], e[7]));
  } else if (p.cache_dt == DSV4_FP4E2M1) {  // e2m1 codes, two per byte, one scale amax/6
    float am = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(e[c]));
    am = group_reduce(am, sh.R, red, true);
    const float scale = am > 0.f ? __fdiv_rn(am, 6.0f) : 1.0f;
    const float inv = am > 0.f ? __fdiv_rn(6.0f, am) : 1.0f;
    if (row) {
      uint32_t w = 0;
#pragma unroll
      for (int c = 0; c < 8; ++c) w |= float_to_e2m1(__fmul_rn(e[c], inv)) << (4 * c);
      *reinterpret_cast<uint32_t *>(static_cast<uint8_t *>(row) + cg * 4) = w;
      if (cg == 0 && sp) *sp = scale;
    }
  } else {
    float am = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) am = fmaxf(am, fabsf(e[c]));
    am = group_reduce(am, sh.R, red, true);
    const float scale = am > 0.f ? __fdiv_rn(am, 448.0f) : 1.0f;
    const float inv = am > 0.f ? __fdiv_rn(448.0f, am) : 1.0f;
    if (row) {
      uint32_t w[2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        w[h] = static_cast<uint32_t>(float2_to_e4m3x2(__fmul_rn(e[4 * h], inv), __fmul_rn(e[4 * h + 1], inv))) |
               (static_cast<uint32_t>(float2_to_e4m3x2(__fmul_rn(e[4 * h + 2], inv), __fmul_rn(e[4 * h + 3], inv)))
                << 16);
      *reinterpret_cast<uint2 *>(static_cast<uint8_t *>(row) + cg * 8) = make_uint2(w[0], w[1]);
      if (cg == 0 && sp) *sp = scale;
    }
  }
  // The state ring keeps each sequence's latest m tokens (slot t % m). The groups that pooled
  // completed blocks stored theirs; the CTA of a sequence's first item (which pooled its first
  // block, the only one that may read ring slots) stores the rest after that: the trailing
  // incomplete block and the slots the first block read.
  __syncthreads();
  for (int k = 0; k < sh.BPC; ++k) {
    const long long it = chunk * sh.BPC + k;
    if (it >= total) break;
    int ss_ = 0;
    int64_t ii = 0;
    SeqRange rr{0, 0, 0};
    map.locate(it, &ss_, &ii, &rr);
    if (ii != 0) continue;  // not the sequence's first item
    float *sst = p.state + static_cast<size_t>(ss_) * p.m * (p.D + p.G);
    const int64_t t0 = rr.p1 - p.m > rr.p0 ? rr.p1 - p.m : rr.p0;
    const int64_t done_end = (rr.p1 / p.m) * p.m;  // tokens below this sit in completed blocks
    const int n = static_cast<int>(rr.p1 - t0);
    // thread -> (token, 8-channel chunk); two tokens' loads in flight before their stores
    constexpr int kTail = 2;
    const int nt = static_cast<int>(blockDim.x);
    for (int base = 0; base < n * sh.R; base += nt * kTail) {
      float v[kTail][8], g[kTail][8];
      int64_t tt[kTail];
      int cc[kTail];
      bool want[kTail];
#pragma unroll
      for (int k2 = 0; k2 < kTail; ++k2) {
        const int e8 = base + k2 * nt + tid;
        tt[k2] = t0 + e8 / sh.R;
        cc[k2] = e8 % sh.R;
        want[k2] = e8 < n * sh.R && (tt[k2] >= done_end || !ring_slot_safe(rr, p.m, tt[k2]));
        if (want[k2]) {
          const TokenSource src{sst, p.kv, p.gate, p.kv_dt, rr.p0, rr.row0, p.m, p.D, p.G};
          load_token8(src, tt[k2], cc[k2], v[k2], g[k2]);
        }
      }
#pragma unroll
      for (int k2 = 0; k2 < kTail; ++k2)
        if (want[k2])
          store_token8(sst + static_cast<size_t>(tt[k2] % p.m) * (p.D + p.G), p.D, p.G, cc[k2], v[k2], g[k2][0], g[k2]);
    }
  }
  __syncthreads();  // the next chunk reuses red and part
}

// prefill items: sequence s owns items [prefix[s], prefix[s + 1])
struct PrefillMap {
  const long long *prefix;
  const int32_t *cu, *start;
  int B;
  __device__ void locate(long long item, int *s, int64_t *i, SeqRange *r) const {
    int lo = 0, hi = B - 1;  // last s with prefix[s] <= item
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= item) lo = mid; else hi = mid - 1;
    }
    *s = lo;
    *i = item - prefix[lo];
    *r = seq_range(cu, start, lo);
  }
};

// Items are the sequences' completed blocks (at least one item per sequence: the state-tail
// write); a CTA takes BPC items at a time (a "chunk"), looping over chunks.
__global__ void __launch_bounds__(kThreads, 2) compress_kernel(const CompressLaunch p) {
  pdl_wait();  // the only kernel of its call: it releases nothing early
  extern __shared__ __align__(16) float smem[];
  const PrefillShape sh = prefill_shape(p.D, p.m);
  float *part = smem;                    // [NG][3][D] partial (max, sum, weighted sum) per slice
  float *red = part + 3 * sh.NG * p.D;   // kThreads / 32
  long long *prefix = reinterpret_cast<long long *>(red + kThreads / 32);  // B + 1
  __shared__ long long warp_tot[kThreads / 32];
  const int tid = threadIdx.x;
  // items before each sequence: a block-wide scan, kThreads sequences per round
  {
    long long carry = 0;
    for (int s0 = 0; s0 < p.B; s0 += kThreads) {
      const int s = s0 + tid;
      const long long c = s < p.B ? compress_items(seq_range(p.cu_seqlens, p.start_pos, s), p.m) : 0;
      long long v = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(0xFFFFFFFFu, v, o);
        if ((tid & 31) >= o) v += u;
      }
      if ((tid & 31) == 31) warp_tot[tid >> 5] = v;
      __syncthreads();
      long long before = carry;
      for (int w = 0; w < (tid >> 5); ++w) before += warp_tot[w];
      if (s < p.B) prefix[s] = before + v - c;
      long long all = carry;
      for (int w = 0; w < kThreads / 32; ++w) all += warp_tot[w];
      carry = all;
      __syncthreads();
    }
    if (tid == 0) prefix[p.B] = carry;
  }
  __syncthreads();
  const long long total = prefix[p.B];
  const long long chunks = (total + sh.BPC - 1) / sh.BPC;
  const CompressView v{p.kv, p.gate, p.kv_dt, p.gamma, p.eps, p.rope_dims, p.rope_theta1, p.state, p.m, p.D, p.G,
                       p.pages, p.scales, p.block_table, p.num_pages, p.max_blocks, p.cache_dt, p.d_status};
  const PrefillMap map{prefix, p.cu_seqlens, p.start_pos, p.B};
  for (long long chunk = blockIdx.x; chunk < chunks; chunk += gridDim.x)
    compress_chunk<false>(v, sh, part, red, chunk, total, map);
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

// decode step: sequence s's one item is the token at pos (input row s)
struct DecodeMap {
  int s;
  int64_t pos;
  __device__ void locate(long long, int *s_out, int64_t *i, SeqRange *r) const {
    *s_out = s;
    *i = 0;
    r->p0 = pos;
    r->p1 = pos + 1;
    r->row0 = s;
  }
};

// One decode step's updates. blockIdx.y: 0 = window insert, 1 = main compressor append,
// 2 = indexer-key compressor append.
// Launched with as few threads as its roles need (a row group per slice of a block: 64 threads
// for D = 512 and m = 4) and little shared memory, so that its CTAs share SMs with the
// indexer's persistent CTAs. In a C4 step it runs beside the indexer, which scores only the
// entries visible before this step's append: it touches nothing the indexer reads, and
// nothing any kernel before it in the call writes. So it releases its dependents at its start
// and waits for its predecessor only at its end (its completion still implies the
// predecessor's: the chain of waits stays unbroken).
__device__ __forceinline__ void decode_prologue_body(const PrologueLaunch &p);

__global__ void __launch_bounds__(kThreads, 2) decode_prologue_kernel(const PrologueLaunch p) {
  pdl_launch_dependents();
  decode_prologue_body(p);
  pdl_wait();
}

__device__ __forceinline__ void decode_prologue_body(const PrologueLaunch &p) {
  extern __shared__ __align__(16) float smem[];  // window role: e[D], red[32]
  float *e = smem;
  float *red = smem + p.D;
  const int s = blockIdx.x, role = blockIdx.y;
  const int tid = threadIdx.x;
  const int64_t pos = p.pos[s];
  if (pos < 0) {
    if (tid == 0) report(p.d_status, DSV4_DEV_BAD_LENGTH);
    return;
  }
  if (role == 0) {
    for (int c = tid; c < p.D; c += static_cast<int>(blockDim.x))
      e[c] = load_one_f(p.kv, p.kv_dt, static_cast<size_t>(s) * p.D + c);
    __syncthreads();
    const size_t slot = static_cast<size_t>(s) * p.W + static_cast<size_t>(pos % p.W);
    void *row = static_cast<char *>(p.ring_rows) + slot * p.D * dtype_size(p.ring_dt);
    finish_and_store(e, p.D, p.gamma, p.eps, pos, p.rope_dims, p.rope_theta1, p.ring_dt, row,
                     p.ring_scales ? p.ring_scales + slot : nullptr, red);
    return;
  }
  // the compressor append of one token per sequence: a one-token prefill at position pos, by
  // the same code (so a token appended here stores what a prefill of it would)
  const bool idx = role == 2;
  const CompressView v{idx ? p.idx_kv : p.kv, idx ? p.idx_gate : p.gate, p.kv_dt, idx ? p.gamma_idx : p.gamma, p.eps,
                       idx ? p.idx_rope_dims : p.rope_dims, idx ? p.idx_rope_theta1 : p.rope_theta1,
                       idx ? p.idx_state : p.state, p.m, idx ? p.idx_D : p.D, idx ? p.idx_G : p.G,
                       idx ? p.idx_pages : p.pages, idx ? p.idx_scales : p.scales,
                       idx ? p.idx_block_table : p.block_table, idx ? p.idx_num_pages : p.num_pages,
                       idx ? p.idx_max_blocks : p.max_blocks, idx ? p.idx_dt : p.cache_dt, p.d_status};
  const PrefillShape sh = prefill_shape(v.D, v.m, static_cast<int>(blockDim.x));
  const DecodeMap map{s, pos};
  // (part, the slices' merge buffer, is only used when a block is split over row groups)
  compress_chunk<true>(v, sh, smem, smem + (sh.S > 1 ? 3 * sh.NG * v.D : 0), 0, 1, map);
}


}  // namespace

cudaError_t launch_compress(const CompressLaunch &p0, cudaStream_t st) {
  CompressLaunch p = p0;
  p.rope_theta1 = rope_theta1(p.rope_base, p.rope_dims);
  const PrefillShape sh = prefill_shape(p.D, p.m);
  const size_t smem = (3 * static_cast<size_t>(sh.NG) * p.D + kThreads / 32) * sizeof(float) +
                      (static_cast<size_t>(p.B) + 1) * sizeof(long long);
  cudaError_t e = cudaFuncSetAttribute(compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // items (blocks, at least one per sequence) are at most total_tokens / m + B; a grid of up to
  // two CTAs per SM loops over chunks of BPC items
  const long long items = static_cast<long long>(p.total_tokens) / p.m + p.B;
  long long grid = (items + sh.BPC - 1) / sh.BPC;
  const long long cap = 2ll * sm_count();
  if (grid > cap) grid = cap;
  return launch_pdl(compress_kernel, dim3(static_cast<unsigned>(grid)), dim3(kThreads), smem, st, 1, p);
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
  // threads: the row groups of one block (each compressor role pools one block); shared
  // memory: the window role's row and reduction slots, or the slices' merge buffer
  int threads = 32;
  size_t floats = static_cast<size_t>(p.D) + 32;
  for (int role = 0; role < (p.idx_D > 0 ? 2 : 1); ++role) {
    const int D = role ? p.idx_D : p.D;
    const PrefillShape sh = prefill_shape(D, p.m);
    const int t = (sh.S * sh.R + 31) / 32 * 32;
    threads = t > threads ? t : threads;
  }
  for (int role = 0; role < (p.idx_D > 0 ? 2 : 1); ++role) {
    const int D = role ? p.idx_D : p.D;
    const PrefillShape sh = prefill_shape(D, p.m, threads);
    const size_t need = (sh.S > 1 ? 3 * static_cast<size_t>(sh.NG) * D : 0) + 32;
    floats = need > floats ? need : floats;
  }
  const size_t smem = floats * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(decode_prologue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.B, p.idx_D > 0 ? 3 : 2);
  return launch_pdl(decode_prologue_kernel, grid, dim3(threads), smem, st, 1, p);
}

}  // namespace dsv4
