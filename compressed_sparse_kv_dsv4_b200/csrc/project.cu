// The compressor's projection (step (1) with its input projection in front; the fused
// "compressor + RMSNorm + RoPE + cache insert" kernel of the vLLM post, SGLang's "Flash
// Compressor" direction): kv_t and gate_t of every new token are its hidden state times the
// compressor's weights, rounded once to bf16, the compressor's input type.
//
//   out[t][c] = bf16( sum_i hidden[t][i] * w[c][i] ),   c < 2 D (kv rows, then gate rows)
//
// A persistent tcgen05 GEMM, one CTA per SM, over 128 x 256 output tiles (tokens x
// channels), in the order that puts the tiles sharing a block of hidden states on
// neighbouring CTAs (so a hidden-state tile is read from DRAM about once and from L2 by the
// others; the weights stay in L2). Warp roles connected by mbarriers:
//   warp 0: TMA of the hidden-state tile [128 x 64] and the weight tile [256 x 64] of each
//           64-wide slice of the hidden dim (bf16, 128B swizzle) into a ring of 4 stages;
//   warp 1: tcgen05.mma kind::f16 (bf16 operands, fp32 accumulation, M = 128, N = 256,
//           K = 16), four per stage, into one of two TMEM accumulators (256 columns each),
//           so the epilogue of one tile overlaps the main loop of the next;
//   warps 2-5: the epilogue, one output row per thread: tcgen05.ld, round to bf16, store
//           the row's 256 channels into kv or gate (rows past the last token are skipped).
// The compressor (compress.cu) then reads kv and gate as its bf16 input.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace dsv4 {

namespace {

constexpr int kPM = 128, kPN = 256, kPK = 64;  // tile: tokens x channels x hidden slice
constexpr int kPStages = 4;
constexpr int kPThreads = 192;
constexpr uint32_t kPStageBytes = (kPM + kPN) * 128;  // bf16 tiles of 64 values per row

struct alignas(1024) ProjSmem {
  uint8_t a[kPStages][kPM * 128];  // hidden states, K-major, 128B swizzle
  uint8_t b[kPStages][kPN * 128];  // weights, K-major, 128B swizzle
  uint64_t full[kPStages], empty[kPStages], acc_full[2], acc_empty[2], mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

struct ProjParams {
  CUtensorMap tmap_h;  // hidden [T][Hd] bf16
  CUtensorMap tmap_w;  // weights [2D][Hd] bf16
  uint16_t *kv;        // [T][D] bf16 bits
  uint16_t *gate;      // [T][D]
  int T, D, Hd;
  int tiles_n;  // 2D / 256
  int tiles;    // ceil(T / 128) * tiles_n
  uint32_t *d_status;
};

__global__ void __launch_bounds__(kPThreads, 1) project_kernel(const __grid_constant__ ProjParams p) {
  extern __shared__ uint8_t smem_raw[];
  ProjSmem &S = *reinterpret_cast<ProjSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    for (int i = 0; i < kPStages; ++i) {
      mbar_init(&S.full[i], 1);
      mbar_init(&S.empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.acc_full[i], 1);
      mbar_init(&S.acc_empty[i], 4);  // the four epilogue warps
    }
    mbar_init(&S.mma_done, 1);
    S.abort_flag = 0;
    fence_mbar_init();
    prefetch_tensormap(&p.tmap_h);
    prefetch_tensormap(&p.tmap_w);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, 2 * kPN);
    tmem_relinquish();
  }
  pdl_wait();  // the hidden states may come from the kernel before
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const int nk = p.Hd / kPK;

  if (warp == 0) {
    // ---------------- producer: stage k of the whole CTA's walk at ring position k % 4
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t lap = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        const int mb = t / p.tiles_n, nb = t % p.tiles_n;
        for (int kb = 0; kb < nk; ++kb) {
          if (issued >= kPStages && !mbar_wait(&S.empty[s], (lap - 1) & 1, &S.abort_flag)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&S.full[s], kPStageBytes);
          tma_load_2d(S.a[s], &p.tmap_h, &S.full[s], kb * kPK, mb * kPM);
          tma_load_2d(S.b[s], &p.tmap_w, &S.full[s], kb * kPK, nb * kPN);
          ++issued;
          if (++s == kPStages) {
            s = 0;
            ++lap;
          }
        }
      }
      if (!ok || S.abort_flag) {  // a role gave up: let the copies in flight land before the CTA leaves
        const int from = issued > kPStages ? kPStages : issued;
        for (int n = from; n >= 1; --n) {
          const int q = issued - n;
          volatile int dummy = 0;
          mbar_wait(&S.full[q % kPStages], static_cast<uint32_t>((q / kPStages) & 1), &dummy);
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: tile j of the CTA into accumulator j % 2
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(kPM, kPN, 0, 0);
      int s = 0, acc = 0, done = 0;
      uint32_t lap = 0, acc_lap = 0;
      bool ok = true, any = false;
      for (int t = blockIdx.x; ok && t < p.tiles; t += gridDim.x) {
        if (done >= 2 && !mbar_wait(&S.acc_empty[acc], (acc_lap - 1) & 1, &S.abort_flag)) break;
        tc_fence_after();
        const uint32_t d = tmem + static_cast<uint32_t>(acc * kPN);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(&S.full[s], lap & 1, &S.abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t ad = sw128_desc(smem_u32(S.a[s]), 16, 1024);
          const uint64_t bd = sw128_desc(smem_u32(S.b[s]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < kPK / 16; ++kk)  // K step of 16 bf16 = 32 bytes = +2 in the descriptor
            mma_bf16(d, ad + 2 * kk, bd + 2 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&S.empty[s]);
          any = true;
          if (++s == kPStages) {
            s = 0;
            ++lap;
          }
        }
        if (!ok) break;
        mma_commit(&S.acc_full[acc]);
        ++done;
        if (++acc == 2) {
          acc = 0;
          ++acc_lap;
        }
      }
      if (any) {  // every MMA issued here completes before the TMEM is freed
        mma_commit(&S.mma_done);
        volatile int dummy = 0;
        mbar_wait(&S.mma_done, 0u, &dummy);
      }
    }
  } else {
    // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. +31 (its rows)
    const int quad = warp & 3;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    int acc = 0;
    uint32_t acc_lap = 0;
    for (int t = blockIdx.x; t < p.tiles; t += gridDim.x) {
      const int mb = t / p.tiles_n, nb = t % p.tiles_n;
      const bool ok = mbar_wait(&S.acc_full[acc], acc_lap & 1, &S.abort_flag);
      if (!__all_sync(0xFFFFFFFFu, ok)) break;
      tc_fence_after();
      const int row = mb * kPM + quad * 32 + lane;
#pragma unroll 1
      for (int c0 = 0; c0 < kPN; c0 += 32) {
        uint32_t r[32];
        tmem_ld32(lane_base + static_cast<uint32_t>(acc * kPN + c0), r);
        tmem_ld_wait();
        const int col = nb * kPN + c0;  // 32 channels of one of kv / gate (D is a multiple of 128)
        uint16_t *dst = col < p.D ? p.kv + static_cast<size_t>(row) * p.D + col
                                  : p.gate + static_cast<size_t>(row) * p.D + (col - p.D);
        if (row < p.T) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 o;
            o.x = pack_bf16x2(__uint_as_float(r[8 * v]), __uint_as_float(r[8 * v + 1]));
            o.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
            o.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
            o.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
            reinterpret_cast<uint4 *>(dst)[v] = o;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.acc_empty[acc]);
      if (++acc == 2) {
        acc = 0;
        ++acc_lap;
      }
    }
  }

  if (tid == 0 && S.abort_flag) report(p.d_status, DSV4_DEV_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 2 * kPN);
  }
}

// bf16 matrix [rows][cols] (row-major), box of 64 columns x box_rows rows, 128B swizzle
bool make_bf16_map(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = get_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols * 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kPK), box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t project_out_bytes(int T, int D) { return align_up(static_cast<size_t>(T) * D * sizeof(uint16_t), 256); }

cudaError_t launch_project(const ProjectLaunch &q, cudaStream_t st) {
  if (q.T <= 0) return cudaSuccess;
  ProjParams p{};
  if (!make_bf16_map(&p.tmap_h, q.hidden, static_cast<uint64_t>(q.T), static_cast<uint64_t>(q.Hd), kPM) ||
      !make_bf16_map(&p.tmap_w, q.w, static_cast<uint64_t>(2 * q.D), static_cast<uint64_t>(q.Hd), kPN))
    return cudaErrorInvalidValue;
  p.kv = q.kv;
  p.gate = q.gate;
  p.T = q.T;
  p.D = q.D;
  p.Hd = q.Hd;
  p.tiles_n = 2 * q.D / kPN;
  p.tiles = (q.T + kPM - 1) / kPM * p.tiles_n;
  p.d_status = q.d_status;
  const size_t smem = sizeof(ProjSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int grid = p.tiles < sm_count() ? p.tiles : sm_count();
  return launch_pdl(project_kernel, dim3(grid), dim3(kPThreads), smem, st, 1, p);
}

}  // namespace dsv4
