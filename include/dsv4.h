/*
 * dsv4.h -- C ABI of a B200 (sm_100a) library for the DeepSeek-V4 hybrid-attention
 * decode step.
 *
 * What the operations are (sources cited by page title and section):
 *  - "Day-0 support for DeepSeek-V4 Pro and Flash on vLLM" (aiwiki entry of the vLLM
 *    announcement), "four moves": shared K/V (V = K) with inverse RoPE on the output,
 *    c4a / c128a KV compression, DeepSeek Sparse Attention over compressed tokens, and a
 *    short sliding window; "vLLM side": one logical block of 256 native positions for
 *    every compression rate, compressor state folded into the SWA cache spec, fused
 *    compressor + RMSNorm + RoPE + cache insert, fp8 attention cache.
 *  - "DeepSeek-V4 launch" review (SGLang/Miles day-0 blog), section "Shadow radix": each
 *    layer is SWA over the latest 128 raw tokens plus C4 (top-512 sparse over 4:1
 *    compressed KV) or C128 (dense over 128:1 compressed KV), with per-layer pools of
 *    in-progress compression state; section "quick overview": Flash Compressor and
 *    Lightning TopK kernels.
 * The pages print no formula. This library computes:
 *  (1) compressor: entry_b = RoPE_{b*m}( RMSNorm( sum_t softmax_t(g_t) * kv_t ) ), the
 *      softmax per channel over the m tokens of block b, then a cache insert;
 *  (2) lightning indexer: s_j = sum_h w_h * ReLU(q_idx_h . k_idx_j), keep the top k;
 *  (3) shared-K/V attention over the selected entries united with the window keys
 *      (or over every entry of a dense C128 layer): o_h = sum_j softmax_j(tau q_h.k_j) k_j,
 *      with q rotated by RoPE_p first;
 *  (4) inverse RoPE: o_h rotated by -p on the rope dims.
 * Conventions (one reading where the pages are silent): RoPE rotates adjacent pairs of the
 * LAST rope_dims dims by pos * base^(-2i/rope_dims); RMSNorm is x/sqrt(mean(x^2)+eps)*gamma;
 * the window key of token t is RoPE_t(RMSNorm(kv_t)) with the compressor's gamma; after
 * token p is appended floor((p+1)/m) entries are visible and the window holds positions
 * max(0,p-W+1)..p; fp8 rows are e4m3 codes with one float32 scale amax/448 per row; top-k
 * ties go to the lower entry index.
 *
 * General rules for every entry point:
 *  - All data pointers are DEVICE pointers owned by the caller (no copies are kept).
 *  - Every call is asynchronous on `stream` (a cudaStream_t); the library never
 *    synchronizes and allocates nothing. Scratch memory is the caller's `workspace` of
 *    at least the size the matching *_workspace_size() returns; it must be 256-byte
 *    aligned and must not be shared by calls that may run concurrently.
 *  - The return value is produced synchronously by host-side validation:
 *    DSV4_ERR_INVALID_ARG (null pointer, misalignment, bad shape), DSV4_ERR_UNSUPPORTED
 *    (a valid combination this build has no kernel for), DSV4_ERR_CUDA (a launch failed).
 *    On any error nothing was launched.
 *  - Faults the device detects (an index or page id out of range, a length beyond the
 *    cache capacity, a bounded wait that gave up) are OR'ed into the caller's device word
 *    *d_status (DSV4_DEV_* bits) and the offending row is skipped; kernels never trap.
 *    d_status may be NULL, in which case such faults are only skipped.
 *  - The library is stateless and thread-safe.
 */
#ifndef DSV4_H
#define DSV4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSV4_ABI_VERSION 3

typedef void *dsv4_stream; /* a cudaStream_t; NULL = the legacy default stream */

typedef enum {
  DSV4_OK = 0,
  DSV4_ERR_INVALID_ARG = 1,
  DSV4_ERR_UNSUPPORTED = 2,
  DSV4_ERR_CUDA = 3,
  DSV4_ERR_SCRATCH_LIMIT = 4 /* the request needs more than the library's static scratch */
} dsv4_status;

/* DSV4_FP4E2M1 ("four moves": "fp4 indexer cache"): OCP e2m1 codes, two per byte (the even
 * element in the low nibble), with one float32 scale amax/6 per row (value = e2m1 * scale).
 * Indexer-key caches only (the keys of dsv4_indexer_topk, a C4 layer's idx_cache, and the cache
 * dsv4_compress writes); a row of dim values is dim/2 bytes. */
typedef enum { DSV4_F32 = 0, DSV4_BF16 = 1, DSV4_FP8E4M3 = 2, DSV4_FP4E2M1 = 3 } dsv4_dtype;

typedef enum { DSV4_LAYER_C4 = 0, DSV4_LAYER_C128 = 1 } dsv4_layer_kind;

/* bits OR'ed into *d_status by the kernels */
#define DSV4_DEV_BAD_INDEX 1u   /* a selected entry index outside [0, n_entries) was skipped */
#define DSV4_DEV_BAD_PAGE 2u    /* a block-table page id outside [0, num_pages) was skipped */
#define DSV4_DEV_TIMEOUT 4u     /* a bounded device wait gave up; results are incomplete */
#define DSV4_DEV_BAD_LENGTH 8u  /* a length or position beyond the cache capacity was clipped */

/* Positions per logical cache block, for every compression rate ("vLLM side": one logical
 * block of 256 native positions). A page of a rate-m cache holds 256/m entries. */
#define DSV4_PAGE_POSITIONS 256

/*
 * Paged cache of compressed entries (or of indexer keys).
 * Entry j of sequence s is row (block_table[s*max_blocks + j/(256/m)], j % (256/m)) of
 * `pages`, laid out [num_pages][256/m][dim] in `dtype` (float32, bfloat16 bits or e4m3
 * codes; rows are contiguous). For DSV4_FP8E4M3, `scales` [num_pages][256/m] holds one
 * float32 per row (value = code * scale); it is ignored (may be NULL) otherwise.
 * m must be a power of two in [1, 256]. `pages` must be 16-byte aligned and dim*size(dtype)
 * a multiple of 16. For DSV4_FP4E2M1 rows are dim/2 bytes with one float32 scale each (scales
 * required); dim/2 must be a multiple of 16.
 */
typedef struct {
  void *pages;
  float *scales;
  const int32_t *block_table; /* [batch][max_blocks] */
  int32_t num_pages;
  int32_t max_blocks;
  int32_t dim;
  int32_t m;
  dsv4_dtype dtype;
} dsv4_paged_cache;

/* Sliding-window ring: position t of sequence s is row (s, t % window) of `rows`
 * [batch][window][dim] in `dtype`; `scales` [batch][window] float32 for DSV4_FP8E4M3. */
typedef struct {
  void *rows;
  float *scales;
  int32_t window;
  int32_t dim;
  dsv4_dtype dtype;
} dsv4_window_ring;

/* Compressor state ("compression-state pool"): the in-progress block of a sequence.
 * buf [batch][m][dim + gate_dim] float32; slot t % m holds token t's kv then its gate. */
typedef struct {
  float *buf;
  int32_t m;
  int32_t dim;
  int32_t gate_dim; /* dim (one gate per channel) or 1 (one gate per token) */
} dsv4_compressor_state;

typedef struct {
  int32_t rope_dims;  /* rotated dims at the end of the vector; even, <= dim; 0 = none */
  float rope_base;    /* theta_i = rope_base^(-2i/rope_dims) */
} dsv4_rope;

/* ------------------------------------------------------------------------------------
 * dsv4_compress: prefill / append of new tokens into one compressor (step (1); vLLM
 * "fused compressor + RMSNorm + RoPE + cache insert", SGLang "Flash Compressor").
 * Sequence s brings tokens kv[cu_seqlens[s] .. cu_seqlens[s+1]) at positions
 * start_pos[s], start_pos[s]+1, ... Every block whose last position is among them is
 * pooled (tokens before start_pos[s] come from `state`), RMS-normed with gamma, rotated
 * by RoPE at position b*m, rounded to the cache dtype and written as entry b. The tokens
 * of a trailing incomplete block are stored in `state`.
 *   kv   [total_tokens][state.dim] in kv_dtype (DSV4_F32 or DSV4_BF16)
 *   gate [total_tokens][state.gate_dim] in kv_dtype
 *   cu_seqlens [batch+1], start_pos [batch]: device int32
 *   gamma [state.dim] float32
 * No workspace. The cache must have room: entry floor((start_pos+len)/m)-1 < max_blocks*256/m.
 */
typedef struct {
  int32_t batch;
  int32_t total_tokens;
  const void *kv;
  const void *gate;
  dsv4_dtype kv_dtype;
  const int32_t *cu_seqlens;
  const int32_t *start_pos;
  const float *gamma;
  float eps;
  dsv4_rope rope;
  dsv4_compressor_state state;
  dsv4_paged_cache cache;
  uint32_t *d_status;
} dsv4_compress_args;

dsv4_status dsv4_compress(const dsv4_compress_args *args, dsv4_stream stream);

/* ------------------------------------------------------------------------------------
 * dsv4_compress_project: dsv4_compress with the compressor's input projection in front
 * (the projection GEMM of the fused compressor: vLLM "compressor + RMSNorm + RoPE + cache
 * insert", SGLang "Flash Compressor"). The kv and gate of token t are its hidden state times
 * the projection weights, each rounded once to bf16 (reading R24):
 *   kv[t][c]   = bf16( sum_i hidden[t][i] * w[c][i] )          c < dim
 *   gate[t][c] = bf16( sum_i hidden[t][i] * w[dim + c][i] )    (one gate per channel)
 * computed on the tensor cores (bf16 operands, fp32 accumulation, one rounding to bf16),
 * then compressed exactly as dsv4_compress with kv_dtype = DSV4_BF16.
 *   c             the compressor arguments; c.kv, c.gate and c.kv_dtype are ignored;
 *                 c.state.gate_dim must equal c.state.dim, and dim must be a multiple of 128.
 *   hidden        [c.total_tokens][hidden_dim] bf16, 16-byte aligned (caller-owned).
 *   w             [2 * dim][hidden_dim] bf16, 16-byte aligned: the kv rows, then the gate rows.
 *   hidden_dim    a positive multiple of 64.
 * Workspace: dsv4_compress_project_workspace_size() bytes, 256-byte aligned, caller-owned.
 * After the call it holds the projected kv [total_tokens][dim] bf16 at offset 0 and gate
 * [total_tokens][dim] bf16 at offset round_up(total_tokens * dim * 2, 256).
 * Errors as dsv4_compress; DSV4_ERR_UNSUPPORTED for a dim or hidden_dim outside the rules.
 */
typedef struct {
  dsv4_compress_args c;
  const void *hidden;
  const void *w;
  int32_t hidden_dim;
} dsv4_compress_project_args;

size_t dsv4_compress_project_workspace_size(const dsv4_compress_project_args *args);
dsv4_status dsv4_compress_project(const dsv4_compress_project_args *args, void *workspace, size_t workspace_bytes,
                                  dsv4_stream stream);

/* ------------------------------------------------------------------------------------
 * dsv4_swa_insert: window keys of new tokens (vLLM "Q-norm + KV RoPE + K insert", the K
 * part): key_t = RoPE_t(RMSNorm(kv_t) * gamma), rounded to the ring dtype, written at
 * slot t % window. Only the last `window` tokens of each sequence are written.
 *   kv [total_tokens][ring.dim] in kv_dtype; cu_seqlens [batch+1], start_pos [batch].
 */
typedef struct {
  int32_t batch;
  int32_t total_tokens;
  const void *kv;
  dsv4_dtype kv_dtype;
  const int32_t *cu_seqlens;
  const int32_t *start_pos;
  const float *gamma;
  float eps;
  dsv4_rope rope;
  dsv4_window_ring ring;
  uint32_t *d_status;
} dsv4_swa_insert_args;

dsv4_status dsv4_swa_insert(const dsv4_swa_insert_args *args, dsv4_stream stream);

/* ------------------------------------------------------------------------------------
 * dsv4_indexer_topk: lightning indexer + top-k (step (2); "DeepSeek Sparse Attention over
 * compressed tokens", SGLang "Lightning TopK").
 *   s_j = sum_h w_h * ReLU( q_h . k_j ),  j < n_entries[s],
 * q_h = q_scale[s][h] * q_idx[s][h] (fp8) or q_idx[s][h] (f32), k_j the dequantized key.
 * If q_rope_dims > 0 the query is first rotated by RoPE at pos[s] on its last q_rope_dims
 * dims (f32 queries only). Writes idx [batch][k] int32: the k best entries (ties to the lower
 * index) in unspecified order, then -1 padding when n_entries[s] < k. If `scores` is not
 * NULL it receives the matching s_j (-inf for padding).
 *   q_idx [batch][heads][dim] in q_dtype (DSV4_F32 or DSV4_FP8E4M3); q_scale [batch][heads]
 *   float32 (fp8 queries; NULL = 1); w [batch][heads] in w_dtype (F32 or BF16);
 *   keys: paged cache with keys.dim == dim, dtype F32, FP8E4M3 or FP4E2M1;
 *   n_entries [batch] device int32 (<= keys.max_blocks * 256/keys.m);
 *   pos [batch] device int32 (used only when q_rope_dims > 0).
 * fp8 queries and fp8 or fp4 keys with dim 128, heads 32 or 64, m == 4, no query RoPE and
 * batch <= 512 run on the tensor cores (tcgen05 kind::f8f6f4, e4m3 or e2m1 keys against e4m3
 * queries, fed by TMA; fp4 pages must be 32-byte aligned); other shapes run on a CUDA-core
 * kernel.
 * Both give the same entries. On the tensor-core path a second kernel selects each
 * sequence's top k from the streamed scores (one thread-block cluster per sequence) and writes
 * idx in ascending entry order.
 */
typedef struct {
  int32_t batch;
  int32_t heads;
  int32_t dim;
  int32_t k;
  const void *q_idx;
  dsv4_dtype q_dtype;
  const float *q_scale;
  const void *w;
  dsv4_dtype w_dtype;
  dsv4_paged_cache keys;
  const int32_t *n_entries;
  const int32_t *pos;
  int32_t q_rope_dims;
  float rope_base;
  int32_t *idx;
  float *scores;
  uint32_t *d_status;
} dsv4_indexer_args;

size_t dsv4_indexer_workspace_size(const dsv4_indexer_args *args);
dsv4_status dsv4_indexer_topk(const dsv4_indexer_args *args, void *workspace,
                              size_t workspace_bytes, dsv4_stream stream);

/* ------------------------------------------------------------------------------------
 * dsv4_indexer_scores: the lightning indexer's scores alone, without the selection (the first
 * half of dsv4_indexer_topk, for a caller that selects by itself): scores[s * scores_ld + j] =
 * s_j for every j < n_entries[s] (the same values dsv4_indexer_topk selects from; -inf where an
 * entry's page is invalid); the rest of each row is left as it is. Same arguments as
 * dsv4_indexer_topk (idx and the args' scores are not used). The tensor-core shapes only
 * (DSV4_ERR_UNSUPPORTED otherwise). scores: device float32, 16-byte aligned; scores_ld a
 * multiple of 4, at least keys.max_blocks * 256 / keys.m. No workspace.
 */
dsv4_status dsv4_indexer_scores(const dsv4_indexer_args *args, float *scores, int64_t scores_ld,
                                dsv4_stream stream);

/* ------------------------------------------------------------------------------------
 * dsv4_indexer_topk_noalloc: dsv4_indexer_topk on scratch the library owns. The pages have
 * no counterpart to this call: it is a convenience of the library, not a step of the method.
 * Same arguments, kernels and results as dsv4_indexer_topk; no workspace argument.
 *
 * Who it is for: a caller that has no device allocator of its own (a plain C host program
 * driving the library) or that must not call cudaMalloc/cudaFree on its decode loop, where
 * each such call stalls the device and the host. The call itself allocates and frees
 * nothing, on the device or the host.
 *
 * Scratch: one file-scope device array of DSV4_NOALLOC_SCRATCH_BYTES (16 MiB) per device,
 * created with the library's device code when the module loads.
 * Set-up: the first call on a device (with that device current) resolves the array's
 * address once (cudaGetSymbolAddress, which may load the module) and caches the SM count;
 * make that first call before any stream capture begins.
 * Limit: if dsv4_indexer_workspace_size(args) > DSV4_NOALLOC_SCRATCH_BYTES the call returns
 * DSV4_ERR_SCRATCH_LIMIT and launches nothing (use dsv4_indexer_topk with a caller
 * workspace instead). The tensor-core path needs about 4 bytes per cache entry of every
 * sequence: 16 MiB admits about 127 sequences of 32768 entries (a 131072-token context).
 * Zero state: nothing has to start at zero; on the CUDA-core path the per-sequence candidate
 * counts at the head of the scratch are zeroed by the call itself, on `stream`, before its
 * kernels run.
 * Concurrency: the scratch is shared by every call on a device. Calls ordered on one
 * stream are safe; calls that can overlap (different streams, or several host threads
 * without ordering) race on the scratch and give wrong results: serialize them.
 */
#define DSV4_NOALLOC_SCRATCH_BYTES (16u << 20)
dsv4_status dsv4_indexer_topk_noalloc(const dsv4_indexer_args *args, dsv4_stream stream);

/* ------------------------------------------------------------------------------------
 * dsv4_sparse_mqa_decode: shared-K/V multi-query attention of one decode query per
 * sequence (steps (3) and (4)).
 * Keys of sequence s: the window positions max(0, pos-W+1)..pos read from `ring`, united
 * with the compressed entries idx[s][0..k) (entries < 0 are skipped) or, when idx is NULL,
 * every entry 0..n_entries[s)-1 (dense). V = K.
 *   o_h = RoPE_{-pos}( sum_j softmax_j( softmax_scale * RoPE_pos(q_h) . k_j ) * k_j )
 *   q [batch][heads][dim] in q_dtype (F32 or BF16), un-rotated; pos [batch] int32;
 *   out [batch][heads][dim] in out_dtype (F32, BF16 or FP8E4M3); lse [batch][heads] float32
 *   (natural log of the softmax denominator, optional).
 *   softmax_scale <= 0 means 1/sqrt(dim).
 *   q_norm_gamma [dim] float32, optional ("vLLM side": the fused "Q-norm + KV RoPE + K
 *   insert" kernel): each query head is first RMS-normed over its dim values with this
 *   weight and q_norm_eps, before RoPE; NULL: no query norm.
 *   FP8E4M3 output ("vLLM side": the fused "inverse RoPE + fp8 quant" kernel): each head's
 *   output, after its inverse RoPE, is stored in blocks of 128 channels as e4m3 codes with one
 *   float32 scale amax/448 per block (1 if the block is all zero) in out_scales
 *   [batch][heads][dim/128] (value = code * scale); dim must be a multiple of 128.
 * cache and ring share dim and dtype (F32, BF16 or FP8E4M3). BF16/FP8 caches with dim 512
 * and heads 64 run on the tensor cores (tcgen05; bf16 operands for BF16 caches, fp16
 * operands holding the exact e4m3 codes with their row scales for FP8 caches; fp32
 * accumulation); other shapes run on a CUDA-core kernel. A sequence with no key gets a zero
 * output. The tensor-core path's workspace holds the prepared query and the partial outputs
 * its thread-block clusters exchange (batch * (cs - 1) * 128 KiB, cs <= 16 the CTAs per
 * sequence); nothing in it outlives the call.
 */
typedef struct {
  int32_t batch;
  int32_t heads;
  int32_t dim;
  const void *q;
  dsv4_dtype q_dtype;
  const int32_t *pos;
  dsv4_paged_cache cache;
  const int32_t *n_entries;
  const int32_t *idx;
  int32_t k;
  dsv4_window_ring ring;
  float softmax_scale;
  dsv4_rope rope;
  void *out;
  dsv4_dtype out_dtype;
  float *lse;
  uint32_t *d_status;
  const float *q_norm_gamma; /* [dim] or NULL */
  float q_norm_eps;
  float *out_scales;         /* [batch][heads][dim/128] for FP8E4M3 output */
} dsv4_mqa_args;

size_t dsv4_mqa_workspace_size(const dsv4_mqa_args *args);
dsv4_status dsv4_sparse_mqa_decode(const dsv4_mqa_args *args, void *workspace,
                                   size_t workspace_bytes, dsv4_stream stream);

/* ------------------------------------------------------------------------------------
 * dsv4_hybrid_decode: one decode step of one hybrid layer for `batch` sequences, each
 * appending the token at pos[s]. In order:
 *   window insert of the new token; main-compressor append (and, when the block
 *   completes, pool + RMSNorm + RoPE + insert); for C4 layers the indexer-key compressor
 *   append; query RoPE; for C4 layers the indexer + top-k over floor((pos+1)/m) entries;
 *   the shared-K/V attention over the window united with the selected (C4) or all
 *   (C128) entries; inverse RoPE; the output store.
 *   (On the tensor-core path of a C4 layer the indexer's scoring kernel runs first, beside the
 *   state updates, over the entries visible before the append; the top-k kernel scores the
 *   appended entry itself. The results are those of the order above.)
 * The caches, the ring and the compressor states are updated in place. n_c is derived
 * from pos; the caller keeps pos < capacity.
 */
typedef struct {
  dsv4_layer_kind kind;
  int32_t heads;
  int32_t dim;
  int32_t topk;          /* C4 only */
  int32_t idx_heads;     /* C4 only */
  int32_t idx_dim;       /* C4 only */
  dsv4_rope rope;        /* main KV, query and output */
  int32_t idx_rope_dims; /* RoPE dims of the indexer-key compressor (same base) */
  int32_t q_idx_rope;    /* 1: rotate an f32 q_idx by RoPE_pos on its last idx_rope_dims dims */
  float eps;
  float softmax_scale;   /* <= 0: 1/sqrt(dim) */
  const float *gamma;        /* [dim] */
  const float *gamma_idx;    /* [idx_dim], C4 only */
  dsv4_compressor_state state;      /* main compressor, state.m = compression rate */
  dsv4_paged_cache cache;           /* main compressed cache (rate state.m) */
  dsv4_window_ring ring;            /* raw window keys */
  dsv4_compressor_state idx_state;  /* C4 only */
  dsv4_paged_cache idx_cache;       /* C4 only */
  const float *gamma_q;             /* [dim]: query norm weight (eps as above); NULL: none */
} dsv4_layer;

typedef struct {
  int32_t batch;
  const int32_t *pos;     /* [batch] */
  const void *kv;         /* [batch][dim] in kv_dtype */
  const void *gate;       /* [batch][state.gate_dim] */
  const void *idx_kv;     /* [batch][idx_dim], C4 only */
  const void *idx_gate;   /* [batch][idx_state.gate_dim], C4 only */
  dsv4_dtype kv_dtype;    /* F32 or BF16, for all four */
  const void *q;          /* [batch][heads][dim], un-rotated */
  dsv4_dtype q_dtype;
  const void *q_idx;      /* [batch][idx_heads][idx_dim], C4 only */
  dsv4_dtype q_idx_dtype;
  const float *q_idx_scale; /* [batch][idx_heads], fp8 q_idx */
  const void *w;          /* [batch][idx_heads] */
  dsv4_dtype w_dtype;
  void *out;              /* [batch][heads][dim] */
  dsv4_dtype out_dtype;   /* F32, BF16 or FP8E4M3 (128-channel blocks, see dsv4_mqa_args) */
  int32_t *topk_idx;      /* optional [batch][topk]: the selected entries (C4) */
  uint32_t *d_status;
  float *out_scales;      /* [batch][heads][dim/128] for FP8E4M3 output */
} dsv4_step;

size_t dsv4_hybrid_decode_workspace_size(const dsv4_layer *layer, int32_t batch);
dsv4_status dsv4_hybrid_decode(const dsv4_layer *layer, const dsv4_step *step, void *workspace,
                               size_t workspace_bytes, dsv4_stream stream);

/* ------------------------------------------------------------------------------------
 * Host helpers (no device work). */

/* Readable name of a status code (static storage). */
const char *dsv4_status_string(dsv4_status status);

/* DSV4_ABI_VERSION of the loaded library. */
int32_t dsv4_abi_version(void);

/* Number of kernels this library has launched in the calling process so far (every device
 * launch of every entry point, counted on the host when the launch is accepted). The
 * difference of two readings is the number of kernels a stretch of calls launched. */
uint64_t dsv4_launch_count(void);

/* Bytes of cache state one layer keeps for one sequence of `context` tokens (vLLM
 * "four moves" sizing: compressed entries of entry_width values at rate m plus `window`
 * raw rows of window_width values), at bytes_per_value bytes per value. */
uint64_t dsv4_layer_state_bytes(uint64_t context, int32_t m, int32_t entry_width,
                                int32_t window, int32_t window_width, int32_t bytes_per_value);

#ifdef __cplusplus
}
#endif

#endif /* DSV4_H */
