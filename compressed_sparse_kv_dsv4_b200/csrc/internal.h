// Host-side interface between the C ABI (api.cu) and the kernel translation units.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cmath>

#include "../../include/dsv4.h"

namespace dsv4 {

// number of SMs of the current device (cached per device)
int sm_count();

// the driver's cuTensorMapEncodeTiled (null if the driver does not provide it)
PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn();

// RoPE's angle step of pair 1, base^(-2/rope_dims), in float64 on the host; pair i turns by
// pos * theta1^i. The launchers fill the rope_theta1 fields below from it.
inline double rope_theta1(float base, int rope_dims) {
  return rope_dims > 0 ? std::pow(static_cast<double>(base), -2.0 / rope_dims) : 1.0;
}

// ---------------------------------------------------------------- compressor / window
struct CompressLaunch {
  int B;
  int total_tokens;
  const void *kv;
  const void *gate;
  dsv4_dtype kv_dt;
  const int32_t *cu_seqlens;
  const int32_t *start_pos;
  const float *gamma;
  float eps;
  int rope_dims;
  float rope_base;
  double rope_theta1 = 1.0;  // filled by the launcher
  float *state;
  int m, D, G;
  void *pages;
  float *scales;
  const int32_t *block_table;
  int num_pages, max_blocks;
  dsv4_dtype cache_dt;
  uint32_t *d_status;
};
cudaError_t launch_compress(const CompressLaunch &p, cudaStream_t st);

// The compressor's input projection: kv [T][D] and gate [T][D] (bf16) = bf16(hidden . w^T),
// hidden [T][Hd] and w [2D][Hd] bf16 (kv rows, then gate rows). Hd % 64 == 0, D % 128 == 0.
struct ProjectLaunch {
  const void *hidden;
  const void *w;
  uint16_t *kv;
  uint16_t *gate;
  int T, D, Hd;
  uint32_t *d_status;
};
// bytes of one projected [T][D] bf16 array in the workspace (256-byte aligned)
size_t project_out_bytes(int T, int D);
cudaError_t launch_project(const ProjectLaunch &p, cudaStream_t st);

struct SwaLaunch {
  int B;
  int total_tokens;
  const void *kv;
  dsv4_dtype kv_dt;
  const int32_t *cu_seqlens;
  const int32_t *start_pos;
  const float *gamma;
  float eps;
  int rope_dims;
  float rope_base;
  double rope_theta1 = 1.0;  // filled by the launcher
  void *rows;
  float *scales;
  int W, D;
  dsv4_dtype ring_dt;
  uint32_t *d_status;
};
cudaError_t launch_swa_insert(const SwaLaunch &p, cudaStream_t st);

// one decode step's state updates: window insert, compressor append(s)
struct PrologueLaunch {
  int B;
  const int32_t *pos;
  dsv4_dtype kv_dt;
  // main
  const void *kv, *gate;
  const float *gamma;
  float eps;
  int rope_dims;
  float rope_base;
  double rope_theta1 = 1.0, idx_rope_theta1 = 1.0;  // filled by the launcher
  float *state;
  int m, D, G;
  void *pages;
  float *scales;
  const int32_t *block_table;
  int num_pages, max_blocks;
  dsv4_dtype cache_dt;
  void *ring_rows;
  float *ring_scales;
  int W;
  dsv4_dtype ring_dt;
  // indexer-key compressor (idx_D == 0: none)
  const void *idx_kv, *idx_gate;
  const float *gamma_idx;
  int idx_rope_dims;
  float *idx_state;
  int idx_D, idx_G;
  void *idx_pages;
  float *idx_scales;
  const int32_t *idx_block_table;
  int idx_num_pages, idx_max_blocks;
  dsv4_dtype idx_dt;
  uint32_t *d_status;
};
cudaError_t launch_decode_prologue(const PrologueLaunch &p, cudaStream_t st);

// ---------------------------------------------------------------- indexer + top-k
struct IndexerLaunch {
  int B, H, Dq, k;
  const void *q;
  dsv4_dtype q_dt;
  const float *q_scale;
  const void *w;
  dsv4_dtype w_dt;
  const void *k_pages;
  const float *k_scales;
  const int32_t *block_table;
  int num_pages, max_blocks, m;
  dsv4_dtype k_dt;
  const int32_t *n_entries;  // NULL: derived from pos as floor((pos+1)/m)
  const int32_t *pos;
  int q_rope_dims;
  float rope_base;
  double rope_theta1 = 1.0;  // of q_rope_dims; filled by the launcher
  int32_t *idx;
  float *scores;
  uint32_t *d_status;
  // Decode step order (n_entries NULL): the scoring kernel runs before the step's prologue
  // and scores the entries visible before the step's append, floor(pos / m); the top-k
  // kernel, which runs after the prologue, scores the appended entry (floor((pos + 1) / m) - 1,
  // when the step completes a block) from the cache row the prologue wrote, and selects over
  // floor((pos + 1) / m) entries. Tensor-core path only.
  bool before_append = false;
  // Another kernel of the same call follows: the last kernel releases it early. When the
  // indexer ends its call, its last kernel does not (the next call's kernels might read
  // what it writes).
  bool release_next = false;
};
bool indexer_uses_tensor_cores(const IndexerLaunch &p);
size_t indexer_workspace_bytes(const IndexerLaunch &p);
cudaError_t launch_indexer_topk(const IndexerLaunch &p, void *ws, cudaStream_t st);
// the scoring kernel alone (tensor-core path), into scores [B][ld], ld >= the capacity
int64_t indexer_score_capacity(const IndexerLaunch &p);
cudaError_t launch_indexer_scores(const IndexerLaunch &p, float *scores, int64_t ld, cudaStream_t st);
// part 1: the scoring kernel only (tensor-core path); part 2: the top-k only; 0: both
cudaError_t launch_indexer_part(const IndexerLaunch &p, void *ws, cudaStream_t st, int part);

// ---------------------------------------------------------------- sparse / dense MQA
struct MqaLaunch {
  int B, H, D;
  const void *q;
  dsv4_dtype q_dt;
  const int32_t *pos;
  const void *pages;
  const float *scales;
  const int32_t *block_table;
  int num_pages, max_blocks, m;
  dsv4_dtype kv_dt;
  const int32_t *n_entries;  // NULL: derived from pos as floor((pos+1)/m)
  const int32_t *idx;        // NULL: dense
  int k;
  const void *ring_rows;
  const float *ring_scales;
  int W;
  float softmax_scale;
  int rope_dims;
  float rope_base;
  double rope_theta1 = 1.0;  // filled by the launcher
  void *out;
  dsv4_dtype out_dt;
  float *lse;
  uint32_t *d_status;
  const float *q_norm_gamma = nullptr;  // [D]: RMS-norm each query head before RoPE (null: no)
  float q_norm_eps = 0.f;
  float *out_scales = nullptr;          // [B][H][D / 128] for fp8 output
};
constexpr int kOutBlock = 128;  // channels per fp8 output block (one scale each)
bool mqa_uses_tensor_cores(const MqaLaunch &p);
size_t mqa_workspace_bytes(const MqaLaunch &p);
cudaError_t launch_mqa(const MqaLaunch &p, void *ws, cudaStream_t st);
// the two halves of launch_mqa, for callers that schedule other kernels between them:
// the query preparation (tensor-core path only) and the attention
cudaError_t launch_mqa_query(const MqaLaunch &p, void *ws, cudaStream_t st);
cudaError_t launch_mqa_attention(const MqaLaunch &p, void *ws, cudaStream_t st);

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Kernels this library has launched in the process (every launch goes through launch_pdl).
void count_launch();

// Launch with programmatic stream serialization (the kernel's pdl_wait() orders it after
// its predecessor), optionally as clusters of `cluster` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st, int cluster,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = static_cast<unsigned>(cluster);
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
  if (e == cudaSuccess) count_launch();
  return e;
}

}  // namespace dsv4
