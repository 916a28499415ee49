// Device-side helpers shared by the decode-step kernels (sm_100a only).
//
// Number formats, RoPE angles, block/warp reductions, bounded mbarrier waits, and thin
// inline-PTX wrappers over TMA (cp.async.bulk.tensor) and the 5th-generation tensor-core
// instructions (tcgen05.*). Nothing here allocates; nothing traps.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dsv4.h"

namespace dsv4 {

// --------------------------------------------------------------------------------------
// device status word

__device__ __forceinline__ void report(uint32_t *d_status, uint32_t bits) {
  if (d_status) atomicOr(d_status, bits);
}

// --------------------------------------------------------------------------------------
// number formats

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint16_t float_to_bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t *>(&h);
}

// two e4m3 codes (lo byte first) -> two floats (exact)
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t v) {
  __half2_raw h = __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(v), __NV_E4M3);
  return __half22float2(*reinterpret_cast<__half2 *>(&h));
}

// two floats -> two e4m3 codes, round to nearest even, saturating to +-448
__device__ __forceinline__ uint16_t float2_to_e4m3x2(float a, float b) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

// pack two floats as bf16x2 (a in the low half)
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  return static_cast<uint32_t>(float_to_bf16_bits(a)) | (static_cast<uint32_t>(float_to_bf16_bits(b)) << 16);
}

// order-preserving map float -> uint32 (larger float -> larger integer); -0 is folded to +0
__device__ __forceinline__ uint32_t float_order_key(float x) {
  uint32_t u = __float_as_uint(x + 0.0f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float order_key_to_float(uint32_t k) {
  uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

// 64-bit top-k key: score order in the high word, lower entry index wins ties
__device__ __forceinline__ unsigned long long topk_key(float score, uint32_t j) {
  return (static_cast<unsigned long long>(float_order_key(score)) << 32) |
         static_cast<unsigned long long>(0xFFFFFFFFu - j);
}

__device__ __forceinline__ uint32_t topk_key_index(unsigned long long key) {
  return 0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull);
}

// --------------------------------------------------------------------------------------
// RoPE: adjacent pairs of the last `rope_dims` dims, angle = pos * base^(-2i/rope_dims).
// The angle is formed and reduced in double precision, so positions up to 2^20 and
// beyond keep ~1e-10 rad accuracy; the rotation itself is done in float.

// cos and sin of RoPE pair `pair` at position pos: angle = pos * theta1^pair with
// theta1 = base^(-2/rope_dims). The angle is formed in float64 (theta1^pair by binary
// powering, relative error ~1e-15) and reduced to [-pi, pi] by a two-constant Cody-Waite
// step with fused multiply-adds; sin and cos of the reduced angle are taken in float32.
__device__ __forceinline__ void rope_cos_sin(int64_t pos, int pair, double theta1, float *c, float *s) {
  constexpr double kTwoPiHi = 6.283185307179586;       // 2*pi rounded to float64
  constexpr double kTwoPiLo = 2.4492935982947064e-16;  // 2*pi - kTwoPiHi
  constexpr double kInvTwoPi = 0.15915494309189535;
  double th = 1.0, b = theta1;
  for (int e = pair; e; e >>= 1) {
    if (e & 1) th *= b;
    b *= b;
  }
  const double a = static_cast<double>(pos) * th;
  const double k = rint(a * kInvTwoPi);
  const double r = fma(-k, kTwoPiLo, fma(-k, kTwoPiHi, a));
  sincosf(static_cast<float>(r), s, c);
}

// --------------------------------------------------------------------------------------
// programmatic dependent launch: a kernel launched with programmatic stream serialization
// may start while its predecessor on the stream still runs. pdl_wait() returns once every
// prerequisite grid has completed and its memory is visible; before it a kernel may only
// touch data no predecessor writes or reads. Each kernel calls pdl_launch_dependents()
// after its own pdl_wait(), so a kernel's early part only ever overlaps its immediate
// predecessor. Launched without the attribute, both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// 2^x by the hardware approximation (one MUFU op; relative error ~2^-22, far below the
// fp16/bf16 rounding the softmax weights receive next); 2^-inf = 0
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// --------------------------------------------------------------------------------------
// reductions

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

// block-wide sum / max for blockDim.x a multiple of 32 (<= 1024); `red` holds >= 32 floats
__device__ __forceinline__ float block_sum(float v, float *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < nw ? red[lane] : 0.f;
  return warp_sum(t);
}

__device__ __forceinline__ float block_max(float v, float *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = lane < nw ? red[lane] : -INFINITY;
  return warp_max(t);
}

// --------------------------------------------------------------------------------------
// loads of `n` consecutive values of a row in a storage dtype, as floats

template <int N>
__device__ __forceinline__ void load_row_f(const void *base, dsv4_dtype dt, size_t elem_off, float (&out)[N]) {
  if (dt == DSV4_F32) {
    const float *p = static_cast<const float *>(base) + elem_off;
#pragma unroll
    for (int i = 0; i < N; i += 4) {
      float4 v = *reinterpret_cast<const float4 *>(p + i);
      out[i] = v.x; out[i + 1] = v.y; out[i + 2] = v.z; out[i + 3] = v.w;
    }
  } else if (dt == DSV4_BF16) {
    const uint16_t *p = static_cast<const uint16_t *>(base) + elem_off;
#pragma unroll
    for (int i = 0; i < N; i += 8) {
      uint4 v = *reinterpret_cast<const uint4 *>(p + i);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        out[i + 2 * k] = __uint_as_float(w[k] << 16);
        out[i + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
  } else {  // e4m3, unscaled
    const uint8_t *p = static_cast<const uint8_t *>(base) + elem_off;
#pragma unroll
    for (int i = 0; i < N; i += 8) {
      uint2 v = *reinterpret_cast<const uint2 *>(p + i);
      const uint32_t w[2] = {v.x, v.y};
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        float2 a = e4m3x2_to_float2(static_cast<uint16_t>(w[k] & 0xFFFF));
        float2 b = e4m3x2_to_float2(static_cast<uint16_t>(w[k] >> 16));
        out[i + 4 * k] = a.x; out[i + 4 * k + 1] = a.y; out[i + 4 * k + 2] = b.x; out[i + 4 * k + 3] = b.y;
      }
    }
  }
}

// OCP e2m1 (1 sign, 2 exponent bits with bias 1, 1 mantissa bit): code -> value (exact)
__device__ __forceinline__ float e2m1_to_float(uint32_t code) {
  const uint32_t e = (code >> 1) & 3u, m = code & 1u;
  // exponent 0: 0.m (0 or 0.5); otherwise 1.m * 2^(e - 1)
  const float mag = e == 0 ? 0.5f * static_cast<float>(m) : __int_as_float(static_cast<int>((e + 126u) << 23 | m << 22));
  return (code & 8u) ? -mag : mag;
}

// float -> e2m1 code: round to nearest, an exact tie to the even mantissa, saturating at 6; the
// sign is kept (a value rounding to zero gives code 8 when negative). Between the
// representable magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6 the midpoints are .25, .75, 1.25, 1.75,
// 2.5, 3.5, 5; at each the even code (mantissa 0: 0, 1, 2, 4) is the lower one for .25, 1.25,
// 2.5, 5 and the upper one for .75, 1.75, 3.5.
__device__ __forceinline__ uint32_t float_to_e2m1(float x) {
  const float a = fabsf(x);
  const uint32_t mag = (a > 0.25f) + (a >= 0.75f) + (a > 1.25f) + (a >= 1.75f) + (a > 2.5f) + (a >= 3.5f) + (a > 5.0f);
  return mag | (signbit(x) ? 8u : 0u);
}

__device__ __forceinline__ float load_one_f(const void *base, dsv4_dtype dt, size_t off) {
  if (dt == DSV4_F32) return static_cast<const float *>(base)[off];
  if (dt == DSV4_BF16) return bf16_bits_to_float(static_cast<const uint16_t *>(base)[off]);
  if (dt == DSV4_FP4E2M1) {  // element off: byte off / 2, the low nibble for even off
    const uint8_t b = static_cast<const uint8_t *>(base)[off >> 1];
    return e2m1_to_float((off & 1) ? (b >> 4) : (b & 15u));
  }
  uint8_t c = static_cast<const uint8_t *>(base)[off];
  return e4m3x2_to_float2(c).x;
}

// bytes of n consecutive values of a row in `dt` (n even for fp4)
__device__ __forceinline__ size_t dtype_bytes(dsv4_dtype dt, size_t n) {
  return dt == DSV4_F32 ? 4 * n : (dt == DSV4_BF16 ? 2 * n : (dt == DSV4_FP4E2M1 ? n / 2 : n));
}
__device__ __forceinline__ size_t dtype_size(dsv4_dtype dt) { return dt == DSV4_F32 ? 4 : (dt == DSV4_BF16 ? 2 : 1); }

// --------------------------------------------------------------------------------------
// shared-memory addresses, mbarriers with bounded waits

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// A wait gives up after this long; the kernel then records DSV4_DEV_TIMEOUT and winds down.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One probe of the phase (the hardware may hold the thread for a short, implementation-
// defined time before answering false).
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase with the given parity to complete. Returns false (and raises *abort)
// if the wait exceeded kWaitLimitNs or another role already raised *abort. Between polls
// the thread sleeps (32 ns, doubling to 128 ns), so a waiting warp leaves the issue slots
// of its SM sub-partition to the warps doing work; the limit is checked every 16 polls.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  uint32_t ns = 32;
  for (uint32_t i = 1;; ++i) {
    __nanosleep(ns);
    if (ns < 128) ns <<= 1;
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        *abort = 1;
        return false;
      }
    }
  }
}

// shared -> global bulk copy (both addresses 16-byte aligned, bytes a multiple of 16),
// tracked by the issuing thread's bulk async-group
__device__ __forceinline__ void bulk_store(void *gdst, const void *ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
               "r"(bytes)
               : "memory");
}
// wait until every bulk copy this thread issued has completed its writes
__device__ __forceinline__ void bulk_store_wait_all() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group 0;\n\tfence.proxy.async.global;" ::: "memory");
}

// start bringing [src, src + bytes) into L2 (16-byte aligned, bytes a multiple of 16)
__device__ __forceinline__ void bulk_prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 16-byte global -> shared copy (both addresses 16-byte aligned), L2 only
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// one arrival on bar once every earlier cp.async of this thread has landed
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void named_bar_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// --------------------------------------------------------------------------------------
// TMA (no multicast anywhere in this library)

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// 1-D bulk copy global -> shared of `bytes` (a multiple of 16; both addresses 16-byte
// aligned), completing as transaction bytes on bar
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// --------------------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in tensor memory)

// Shared-memory matrix descriptor, 128-byte swizzle (the layout TMA's SWIZZLE_128B writes):
// 8-row x 128-byte atoms, `sbo` bytes between 8-row groups, `lbo` bytes between atoms
// along the leading dimension (MN-major operands; ignored for K-major).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version for sm_100
  d |= static_cast<uint64_t>(2) << 61;  // 128-byte swizzle
  return d;
}

// Instruction descriptors: fp32 accumulate; a_mn/b_mn = 1 for MN-major operands.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// kind::f8f6f4 with A in e2m1 (format 5; in shared memory as 16 values in the first 8 bytes of
// each 16-byte chunk, the layout TMA's 16U4_ALIGN16B type writes) and B in e4m3
__host__ __device__ constexpr uint32_t idesc_e2m1_e4m3(int M, int N) {
  return (1u << 4) | (5u << 7) | (0u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(a_mn) << 15) |
         (static_cast<uint32_t>(b_mn) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// kind::f16 MMA (fp16 or bf16 operands, as the instruction descriptor says)
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}

// the same MMA, issued only when en != 0 (predicated, not branched around: a thread that
// passes en = 0 still goes through the instruction)
__device__ __forceinline__ void mma_bf16_if(uint32_t en, uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\tsetp.ne.b32 e, %5, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(en)
      : "memory");
}

__device__ __forceinline__ void mma_commit_if(uint32_t en, uint64_t *bar) {
  asm volatile(
      "{\n\t.reg .pred e;\n\tsetp.ne.b32 e, %1, 0;\n\t"
      "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}" ::"r"(smem_u32(bar)),
      "r"(en)
      : "memory");
}

// arrive on an mbarrier once every previously issued tcgen05 op of this thread completed
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bits, 32 consecutive columns: thread t of the warp gets lane (base lane + t)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// 16 lanes x 32 bits, twice: thread t of the warp takes lane (base lane + t % 16), and its
// register j is column (base column + 32 (t / 16) + j). Touches only the 16 lanes from the
// base lane, so it leaves the other 16 lanes of the warp's quadrant alone.
__device__ __forceinline__ void tmem_ld16x2(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void tmem_st16x2(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.16x32bx2.x32.b32 [%0], 32, "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

// byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside a 128B-swizzled region
// whose rows are 128 bytes and whose 8-row groups are 1024 bytes apart
__device__ __forceinline__ uint32_t sw128_offset(int row, int chunk) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 + ((chunk ^ (row & 7)) << 4));
}

}  // namespace dsv4
