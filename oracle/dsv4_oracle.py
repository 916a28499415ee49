"""Plain float64 restatement of the DeepSeek-V4 hybrid-attention decode step.

TEST INFRASTRUCTURE ONLY. This module is the oracle the CUDA library is
checked against. Only the tests, the smoke check and the CPU-baseline /
reference arm of the benchmark may import it; the library never does, and
nothing here imports the library. It is deliberately slow: every step is
written the way the method states it, in float64, with plain numpy.

Sources, cited by page title and section:

[vLLM]   "Day-0 support for DeepSeek-V4 Pro and Flash on vLLM" (the vLLM
         announcement as quoted by the aiwiki entry).
         - "four moves" list: shared K/V + inverse RoPE; c4a / c128a KV
           compression; DeepSeek Sparse Attention over compressed tokens; short
           sliding window for locality across compression boundaries.
         - "vLLM side" list: unified hybrid KV cache with one logical block of
           256 native positions for every compression rate; compressor state
           folded into the SWA KV-cache spec; fused "compressor + RMSNorm +
           RoPE + cache insert", "inverse RoPE + fp8 quant" and "Q-norm + KV
           RoPE + K insert" kernels; fp8 attention cache.
         - the KV-state sizing sentence (9.62 GiB vs 83.9 GiB at 1M context).
[SGLang] "DeepSeek-V4 launch" review (winzheng.jp, a translation of the
         SGLang/Miles day-0 blog), section "Shadow radix": every layer pairs
         SWA over the latest 128 raw tokens with either C4 (top-512 sparse over
         4:1 compressed KV) or C128 (dense over 128:1 compressed KV), and each
         compressed layer keeps a pool of in-progress compression state.
[NVIDIA] "DeepSeek-V4 auf NVIDIA Blackwell und GPU-beschleunigten Endpoints
         verfuegbar" (ki-news-radar.de): CSA (compressed sparse attention, C4
         + DSA) and HCA (heavily compressed attention, C128) naming.

The pages name these parts but print no formula. The problem statement this
library implements fixes four of them:
  (1) compressor: softmax-gated weighted pool of the block's projected KV,
      then RMSNorm, then RoPE at the block's position, then cache insert;
  (2) lightning indexer: s_j = sum_h w_h * ReLU(q_idx_h . k_idx_j), keep the
      top-k (k = 512 in the C4 layers);
  (3) shared-K/V (V = K) multi-query attention over the selected compressed
      entries united with a 128-token sliding window of raw tokens, or over all
      entries of a dense C128 layer;
  (4) inverse RoPE: rotate the output by -pos_q on the rope dims.

Readings taken where both are silent (the plainest one the text supports):
  R1  gate width: one gate logit per channel (G = D); a scalar gate per token
      (G = 1) is the broadcast special case.
  R2  the gating softmax runs over the m tokens of a block, per channel, with
      the maximum subtracted first; no positional bias.
  R3  blocks do not overlap: block b holds positions [b*m, (b+1)*m).
  R4  the raw window key of token t is RoPE_t(RMSNorm(kv_t)) with the same
      norm weight as the compressor.
  R5  RMSNorm over all D dims: x / sqrt(mean(x^2) + eps) * gamma.
  R6  RoPE rotates adjacent pairs (x[D-r+2i], x[D-r+2i+1]) of the LAST r
      dims by angle pos * theta_i, theta_i = base^(-2i/r).
  R7  a block's position is b*m (its first raw position).
  R8  the query is rotated by RoPE_p before the logits.
  R9  after the decode token p is appended, n_c = floor((p+1)/m) entries are
      visible; the window holds positions max(0, p-W+1) .. p (the current token
      included); entries overlapping the window are not masked.
  R10 one shared indexer key per C4 entry, built by its own compressor.
  R11 head weights w are an input per query; no softmax, no extra scale.
  R12 fp8 caches: e4m3 codes with one float32 scale per entry,
      scale = amax/448 (1 when amax = 0), code = RNE_satfinite(x * (448/amax))
      with the division and the product rounded to float32.
  R13 softmax scale 1/sqrt(D) over all D dims; no attention sinks.
  R14 top-k ties go to the lower entry index; with n_c <= k every entry is
      taken and the rest of the k slots hold -1.
  R15 with no visible key at all the output is zero.
  R21 query norm ([vLLM] "vLLM side": the fused "Q-norm + KV RoPE + K insert"
      kernel): when a layer has a query norm weight, each query head is
      RMS-normed over its D dims with that weight and the layer's eps before its
      RoPE, like the window key of R4.
  R23 fp4 indexer cache ([vLLM] "four moves": "fp8 attention cache + fp4
      indexer cache"): an fp4 row is OCP e2m1 codes (1 sign, 2 exponent bits
      with bias 1, 1 mantissa bit: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6), two
      per byte with the even element in the low nibble, plus one float32 scale
      amax/6 per row (1 if amax = 0); code = RNE_satfinite(x * (6/amax)), the
      rule of R12 with 6 the largest e2m1 magnitude.
  R24 projection in front of the compressor ([vLLM] "vLLM side" fuses the
      compressor with its cache insert; SGLang's "Flash Compressor"): kv_t and
      gate_t are the products of token t's hidden state with the compressor's
      projection weights (kv rows, then gate rows), each rounded once to bf16,
      the compressor's input type (nearest, ties to even, from the exact value).
  R22 fp8 output ([vLLM] "vLLM side": the fused "inverse RoPE + fp8 quant"
      kernel): the output of each head, after its inverse RoPE, is stored as
      e4m3 codes in blocks of 128 channels, each block with one float32 scale
      amax/448 (the rule of R12 applied to every 128-value block).
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

PAGE_POSITIONS = 256  # [vLLM] "vLLM side": one logical block = 256 native positions

# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------
# OCP 8-bit floating point, E4M3 variant: 1 sign bit, 4 exponent bits with
# bias 7, 3 mantissa bits, no infinities, S.1111.111 = NaN, largest finite 448.

E4M3_MAX = 448.0


def _e4m3_value(code: int) -> float:
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return float("nan")
    if exp == 0:  # subnormal: 0.mmm * 2^(1-bias)
        return sign * (man / 8.0) * 2.0 ** (1 - 7)
    return sign * (1.0 + man / 8.0) * 2.0 ** (exp - 7)


E4M3_VALUES = np.array([_e4m3_value(c) for c in range(256)], dtype=np.float64)
_E4M3_POS = E4M3_VALUES[:0x7F]  # codes 0x00..0x7E: 0 .. 448, increasing


def e4m3_decode(codes) -> np.ndarray:
    """e4m3 codes (uint8) -> float64 values, from the format definition."""
    return E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """float32 values -> e4m3 codes, round to nearest (ties to even), saturating.

    Finite inputs only. |x| > 448 saturates to 448 (the 'satfinite' rule), and
    a value that rounds to zero keeps its sign (0x80 for negatives).
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode: non-finite input")
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.minimum(np.searchsorted(_E4M3_POS, a, side="left"), 0x7E)
    lo = np.maximum(hi - 1, 0)
    d_hi = _E4M3_POS[hi] - a
    d_lo = a - _E4M3_POS[lo]
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(take_hi, hi, lo).astype(np.uint8)
    return mag | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)


# OCP 4-bit floating point, E2M1: 1 sign bit, 2 exponent bits with bias 1, 1
# mantissa bit, no infinities or NaN, largest finite 6 (reading R23).

E2M1_MAX = 6.0


def _e2m1_value(code: int) -> float:
    sign = -1.0 if code & 0x8 else 1.0
    exp = (code >> 1) & 0x3
    man = code & 0x1
    if exp == 0:  # subnormal: 0.m * 2^(1-bias)
        return sign * (man / 2.0)
    return sign * (1.0 + man / 2.0) * 2.0 ** (exp - 1)


E2M1_VALUES = np.array([_e2m1_value(c) for c in range(16)], dtype=np.float64)
_E2M1_POS = E2M1_VALUES[:8]  # codes 0..7: 0 .. 6, increasing


def e2m1_decode(codes) -> np.ndarray:
    """e2m1 codes (0..15) -> float64 values, from the format definition."""
    return E2M1_VALUES[np.asarray(codes, dtype=np.uint8) & 0xF]


def e2m1_encode(x) -> np.ndarray:
    """float32 values -> e2m1 codes (0..15): round to nearest, ties to the even
    mantissa, saturating at 6; a value rounding to zero keeps its sign (code 8)."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("e2m1_encode: non-finite input")
    a = np.minimum(np.abs(x), E2M1_MAX)
    hi = np.minimum(np.searchsorted(_E2M1_POS, a, side="left"), 7)
    lo = np.maximum(hi - 1, 0)
    d_hi = _E2M1_POS[hi] - a
    d_lo = a - _E2M1_POS[lo]
    take_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(take_hi, hi, lo).astype(np.uint8)
    return mag | np.where(np.signbit(x), 0x8, 0).astype(np.uint8)


def fp4_pack(codes) -> np.ndarray:
    """e2m1 codes [..., D] -> bytes [..., D/2], element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def fp4_unpack(packed) -> np.ndarray:
    """bytes [..., D/2] -> e2m1 codes [..., D]."""
    b = np.asarray(packed, dtype=np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = b & 0xF
    out[..., 1::2] = b >> 4
    return out


def bf16_decode(bits) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> float64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def bf16_encode(x) -> np.ndarray:
    """float32 -> bfloat16 bits, round to nearest even on the 16 dropped bits."""
    u = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def f32(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32)


# ---------------------------------------------------------------------------
# the per-vector steps
# ---------------------------------------------------------------------------

def rope_inv_freq(rope_dims: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/r), i = 0 .. r/2-1 (reading R6)."""
    i = np.arange(rope_dims // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / float(rope_dims))


def apply_rope(x, pos: int, rope_dims: int, base: float, inverse: bool = False) -> np.ndarray:
    """Rotate adjacent pairs of the last `rope_dims` dims of x by pos*theta_i.

    inverse=True rotates by -pos*theta_i ([vLLM] "four moves": inverse RoPE on
    the output, needed because V = K carries the rotation).
    """
    y = np.array(x, dtype=np.float64, copy=True)
    if rope_dims == 0:
        return y
    d = y.shape[-1]
    ang = float(pos) * rope_inv_freq(rope_dims, base)
    if inverse:
        ang = -ang
    c, s = np.cos(ang), np.sin(ang)
    x0 = y[..., d - rope_dims::2].copy()
    x1 = y[..., d - rope_dims + 1::2].copy()
    y[..., d - rope_dims::2] = x0 * c - x1 * s
    y[..., d - rope_dims + 1::2] = x0 * s + x1 * c
    return y


def rms_norm(x, gamma, eps: float) -> np.ndarray:
    """x / sqrt(mean(x^2) + eps) * gamma over the last axis (reading R5)."""
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(gamma, np.float64)


def gated_pool(kv_block, gate_block) -> np.ndarray:
    """Softmax-gated pool of one block (readings R1, R2).

    kv_block [m, D], gate_block [m, G] with G in {1, D}:
    e_c = sum_t softmax_t(g_{t,c}) * kv_{t,c}.
    """
    kv = np.asarray(kv_block, dtype=np.float64)
    g = np.broadcast_to(np.asarray(gate_block, dtype=np.float64), kv.shape)
    e = np.exp(g - g.max(axis=0, keepdims=True))
    return (e / e.sum(axis=0, keepdims=True) * kv).sum(axis=0)


def compress_block(kv_block, gate_block, block_index: int, m: int, gamma, eps: float,
                   rope_dims: int, rope_base: float) -> np.ndarray:
    """Step (1): pool -> RMSNorm -> RoPE at the block position b*m (R7)."""
    e = gated_pool(kv_block, gate_block)
    e = rms_norm(e, gamma, eps)
    return apply_rope(e, block_index * m, rope_dims, rope_base)


def window_key(kv_t, pos: int, gamma, eps: float, rope_dims: int, rope_base: float) -> np.ndarray:
    """Raw sliding-window key of token `pos` (reading R4)."""
    return apply_rope(rms_norm(kv_t, gamma, eps), pos, rope_dims, rope_base)


def store(x, dtype: str):
    """Round a float64 vector into a cache dtype the way the cache stores it.

    Returns (codes, scale, decoded float64). f32: float32 values; bf16: bits;
    fp8: e4m3 codes with one float32 scale (reading R12).
    """
    x32 = f32(x)
    if dtype == "f32":
        return x32, np.float32(1.0), x32.astype(np.float64)
    if dtype == "bf16":
        b = bf16_encode(x32)
        return b, np.float32(1.0), bf16_decode(b)
    if dtype == "fp8":
        amax = np.float32(np.max(np.abs(x32)))
        if amax == 0:
            scale = np.float32(1.0)
            inv = np.float32(1.0)
        else:
            scale = np.float32(amax / np.float32(E4M3_MAX))
            inv = np.float32(np.float32(E4M3_MAX) / amax)
        codes = e4m3_encode((x32 * inv).astype(np.float32))
        return codes, scale, e4m3_decode(codes) * np.float64(scale)
    if dtype == "fp4":  # reading R23: packed e2m1 codes, one scale amax/6
        amax = np.float32(np.max(np.abs(x32)))
        if amax == 0:
            scale = np.float32(1.0)
            inv = np.float32(1.0)
        else:
            scale = np.float32(amax / np.float32(E2M1_MAX))
            inv = np.float32(np.float32(E2M1_MAX) / amax)
        codes = e2m1_encode((x32 * inv).astype(np.float32))
        return fp4_pack(codes), scale, e2m1_decode(codes) * np.float64(scale)
    raise ValueError(dtype)


def decode_rows(codes, scales, dtype: str) -> np.ndarray:
    """Stored rows [..., D] (+ per-row scales [...]) -> float64."""
    if dtype == "f32":
        return np.asarray(codes, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_decode(codes)
    if dtype == "fp8":
        return e4m3_decode(codes) * np.asarray(scales, dtype=np.float32).astype(np.float64)[..., None]
    if dtype == "fp4":
        return e2m1_decode(fp4_unpack(codes)) * np.asarray(scales, dtype=np.float32).astype(np.float64)[..., None]
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# caches and state (the same byte layout the library uses)
# ---------------------------------------------------------------------------

CODE_DTYPE = {"f32": np.float32, "bf16": np.uint16, "fp8": np.uint8, "fp4": np.uint8}


@dataclass
class PagedCache:
    """Compressed-entry cache: pages of 256 native positions ([vLLM] "vLLM side").

    A page holds 256/m entries. Entry j of sequence s lives in physical page
    block_table[s, j // (256/m)] at slot j % (256/m).
    """
    dtype: str
    m: int
    D: int
    pages: np.ndarray        # [num_pages, 256 // m, D] codes ([.., D/2] bytes for fp4)
    scales: np.ndarray       # [num_pages, 256 // m] float32 (fp8; ones otherwise)
    block_table: np.ndarray  # [B, max_blocks] int32

    @property
    def per_page(self) -> int:
        return PAGE_POSITIONS // self.m

    def locate(self, s: int, j):
        j = np.asarray(j, dtype=np.int64)
        return self.block_table[s, j // self.per_page], j % self.per_page

    def read(self, s: int, j) -> np.ndarray:
        pg, sl = self.locate(s, j)
        return decode_rows(self.pages[pg, sl], self.scales[pg, sl], self.dtype)

    def write(self, s: int, j: int, x) -> None:
        pg, sl = self.locate(s, j)
        codes, scale, _ = store(x, self.dtype)
        self.pages[pg, sl] = codes
        self.scales[pg, sl] = scale


@dataclass
class WindowRing:
    """Sliding-window cache: W slots per sequence, position t at slot t % W."""
    dtype: str
    W: int
    D: int
    rows: np.ndarray    # [B, W, D] codes
    scales: np.ndarray  # [B, W] float32

    def write(self, s: int, pos: int, x) -> None:
        codes, scale, _ = store(x, self.dtype)
        self.rows[s, pos % self.W] = codes
        self.scales[s, pos % self.W] = scale

    def read(self, s: int, positions) -> np.ndarray:
        slots = np.asarray(positions, dtype=np.int64) % self.W
        return decode_rows(self.rows[s, slots], self.scales[s, slots], self.dtype)


@dataclass
class CompressorState:
    """In-progress block of one compressor ([SGLang] "Shadow radix": state pools).

    buf[s, t % m] holds (kv_t, gate_t) of token t as float32, kv first.
    """
    m: int
    D: int
    G: int
    buf: np.ndarray  # [B, m, D + G] float32


def compress_tokens(state: CompressorState, cache: PagedCache, s: int, start_pos: int,
                    kv, gate, gamma, eps: float, rope_dims: int, rope_base: float) -> None:
    """Feed tokens start_pos, start_pos+1, ... of sequence s into the compressor.

    Each token is stored in its ring slot; when the slot is the last of a block
    (t % m == m-1) the block is complete and its entry is pooled, normed,
    rotated and written to the paged cache at entry index t // m.
    """
    m, d = state.m, state.D
    kv = np.asarray(kv, dtype=np.float64)
    gate = np.asarray(gate, dtype=np.float64).reshape(kv.shape[0], -1)
    for i in range(kv.shape[0]):
        t = start_pos + i
        slot = t % m
        state.buf[s, slot, :d] = kv[i]
        state.buf[s, slot, d:] = gate[i]
        if slot == m - 1:
            blk = state.buf[s].astype(np.float64)
            entry = compress_block(blk[:, :d], blk[:, d:], t // m, m, gamma, eps, rope_dims, rope_base)
            cache.write(s, t // m, entry)


def bf16_round_exact(x) -> np.ndarray:
    """float64 -> the nearest bf16 value (8 significant bits), ties to even, as float64:
    one rounding from the given value (no intermediate float32)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)  # x = m * 2^e, 0.5 <= |m| < 1
    return np.ldexp(np.round(np.ldexp(m, 8)), e - 8)  # np.round: half to even


def project(hidden, w, dim: int):
    """R24: kv = bf16(hidden . w[:dim]^T), gate = bf16(hidden . w[dim:]^T), each element
    rounded once from its exact (float64) dot product. hidden [T, Hd], w [2 dim, Hd] as
    values; returns (kv, gate) as bf16 bits [T, dim]."""
    h = np.asarray(hidden, dtype=np.float64)
    wt = np.asarray(w, dtype=np.float64)
    out = bf16_round_exact(h @ wt.T)
    bits = bf16_encode(out.astype(np.float32))  # exact: every value is a bf16 value
    return bits[:, :dim], bits[:, dim:]


def compress(kv, gate, cu_seqlens, start_pos, state: CompressorState, cache: PagedCache,
             gamma, eps: float, rope_dims: int, rope_base: float) -> None:
    """Prefill: sequence s brings tokens kv[cu[s]:cu[s+1]] at positions start_pos[s].."""
    for s in range(len(cu_seqlens) - 1):
        a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        compress_tokens(state, cache, s, int(start_pos[s]), kv[a:b], gate[a:b], gamma, eps,
                        rope_dims, rope_base)


def swa_insert(ring: WindowRing, s: int, pos: int, kv_t, gamma, eps: float, rope_dims: int,
               rope_base: float) -> None:
    ring.write(s, pos, window_key(kv_t, pos, gamma, eps, rope_dims, rope_base))


# ---------------------------------------------------------------------------
# indexer, top-k, attention
# ---------------------------------------------------------------------------

def indexer_scores(q_idx, w, keys) -> np.ndarray:
    """s_j = sum_h w_h * ReLU(q_h . k_j)   (step (2), reading R11).

    q_idx [H_I, d_I], w [H_I], keys [n, d_I] -> s [n], all float64.
    """
    dots = np.asarray(keys, np.float64) @ np.asarray(q_idx, np.float64).T  # [n, H_I]
    return np.maximum(dots, 0.0) @ np.asarray(w, np.float64)


def topk_select(scores, k: int) -> np.ndarray:
    """The k largest scores, ties to the lower index (R14); -1 pads when n < k.

    Returned in (score descending, index ascending) order.
    """
    s = np.asarray(scores, dtype=np.float64)
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))[: min(k, n)]
    out = np.full(k, -1, dtype=np.int64)
    out[: order.shape[0]] = order
    return out


def shared_kv_attention(q, pos: int, keys, softmax_scale: float, rope_dims: int,
                        rope_base: float) -> np.ndarray:
    """Steps (3)+(4): V = K attention over `keys`, then inverse RoPE.

    q [H, D] un-rotated query; keys [N, D] already carry their own rotations.
    o_h = RoPE_{-p}( sum_j softmax_j(tau * RoPE_p(q_h) . k_j) * k_j ).
    """
    keys = np.asarray(keys, dtype=np.float64)
    h, d = np.shape(q)
    if keys.shape[0] == 0:
        return np.zeros((h, d))
    qr = apply_rope(q, pos, rope_dims, rope_base)
    logits = softmax_scale * (qr @ keys.T)
    logits -= logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p /= p.sum(axis=1, keepdims=True)
    return apply_rope(p @ keys, pos, rope_dims, rope_base, inverse=True)


def query_norm(q, gamma_q, eps: float) -> np.ndarray:
    """R21: each head of q [H, D] RMS-normed over its D dims, times gamma_q [D]."""
    return rms_norm(q, gamma_q, eps)


OUT_BLOCK = 128  # channels per fp8 output block (R22)


def store_output(o, dtype: str):
    """Round an attention output [H, D] into its stored form (R22 for fp8).

    Returns (codes, scales, decoded float64): f32 / bf16 rows as `store` gives
    them (scales [H, 1] of ones); fp8: codes [H, D] and scales [H, D/128], each
    128-channel block rounded by `store` on its own.
    """
    o = np.asarray(o, dtype=np.float64)
    h, d = o.shape
    if dtype != "fp8":
        codes, _, dec = store(o, dtype)
        return codes, np.ones((h, 1), np.float32), dec
    nb = d // OUT_BLOCK
    codes = np.zeros((h, d), np.uint8)
    scales = np.zeros((h, nb), np.float32)
    dec = np.zeros((h, d))
    for i in range(h):
        for j in range(nb):
            sl = slice(j * OUT_BLOCK, (j + 1) * OUT_BLOCK)
            codes[i, sl], scales[i, j], dec[i, sl] = store(o[i, sl], "fp8")
    return codes, scales, dec


def window_positions(pos: int, W: int) -> np.ndarray:
    """Positions max(0, p-W+1) .. p (reading R9)."""
    return np.arange(max(0, pos - W + 1), pos + 1, dtype=np.int64)


def visible_entries(pos: int, m: int) -> int:
    """n_c = floor((p+1)/m) complete blocks once token p is in (reading R9)."""
    return (pos + 1) // m


# ---------------------------------------------------------------------------
# one layer, one decode step
# ---------------------------------------------------------------------------

@dataclass
class LayerConfig:
    kind: str            # "c4" (CSA: indexer + top-k) or "c128" (HCA: dense)
    m: int
    H: int
    D: int
    W: int = 128
    k: int = 512
    H_I: int = 0
    d_I: int = 0
    rope_dims: int = 64
    rope_base: float = 10000.0
    idx_rope_dims: int = 0   # RoPE dims of the indexer-key compressor
    q_idx_rope: bool = False  # rotate q_idx by RoPE_p on its last idx_rope_dims dims
    eps: float = 1e-6
    softmax_scale: float = 0.0  # 0 -> 1/sqrt(D)

    @property
    def tau(self) -> float:
        return self.softmax_scale if self.softmax_scale > 0 else 1.0 / np.sqrt(self.D)


@dataclass
class LayerState:
    cfg: LayerConfig
    gamma: np.ndarray
    main_state: CompressorState
    main_cache: PagedCache
    window: WindowRing
    gamma_idx: np.ndarray | None = None
    idx_state: CompressorState | None = None
    idx_cache: PagedCache | None = None
    gamma_q: np.ndarray | None = None  # query norm weight (R21); None: no query norm


@dataclass
class StepInputs:
    """Per-sequence inputs of one decode step, decoded to float64."""
    pos: np.ndarray           # [B] int
    kv: np.ndarray            # [B, D]
    gate: np.ndarray          # [B, G]
    q: np.ndarray             # [B, H, D]  un-rotated
    q_idx: np.ndarray | None = None   # [B, H_I, d_I]
    w: np.ndarray | None = None       # [B, H_I]
    idx_kv: np.ndarray | None = None  # [B, d_I]
    idx_gate: np.ndarray | None = None


def decode_update(layer: LayerState, step: StepInputs) -> None:
    """State updates of one decode step: window insert, compressor append(s)."""
    c = layer.cfg
    for s in range(step.pos.shape[0]):
        p = int(step.pos[s])
        swa_insert(layer.window, s, p, step.kv[s], layer.gamma, c.eps, c.rope_dims, c.rope_base)
        compress_tokens(layer.main_state, layer.main_cache, s, p, step.kv[s:s + 1],
                        step.gate[s:s + 1], layer.gamma, c.eps, c.rope_dims, c.rope_base)
        if c.kind == "c4":
            compress_tokens(layer.idx_state, layer.idx_cache, s, p, step.idx_kv[s:s + 1],
                            step.idx_gate[s:s + 1], layer.gamma_idx, c.eps, c.idx_rope_dims,
                            c.rope_base)


def select_entries(layer: LayerState, step: StepInputs, s: int):
    """Entry indices attended by sequence s: top-k (C4) or all (C128)."""
    c = layer.cfg
    p = int(step.pos[s])
    n_c = visible_entries(p, c.m)
    if c.kind != "c4":
        return np.arange(n_c, dtype=np.int64), None
    q_idx = np.asarray(step.q_idx[s], dtype=np.float64)
    if c.q_idx_rope:
        q_idx = apply_rope(q_idx, p, c.idx_rope_dims, c.rope_base)
    if n_c == 0:
        return np.zeros(0, dtype=np.int64), np.zeros(0)
    keys = layer.idx_cache.read(s, np.arange(n_c))
    scores = indexer_scores(q_idx, step.w[s], keys)
    idx = topk_select(scores, c.k)
    return idx[idx >= 0], scores


def decode_attend(layer: LayerState, step: StepInputs, seqs=None):
    """Attention part of one decode step, for the sequences in `seqs`.

    Returns {s: (o [H, D], selected entry indices, indexer scores or None)}.
    """
    c = layer.cfg
    out = {}
    for s in (range(step.pos.shape[0]) if seqs is None else seqs):
        p = int(step.pos[s])
        sel, scores = select_entries(layer, step, s)
        parts = [layer.window.read(s, window_positions(p, c.W))]
        if sel.shape[0]:
            parts.append(layer.main_cache.read(s, sel))
        keys = np.concatenate(parts, axis=0)
        q = step.q[s]
        if layer.gamma_q is not None:
            q = query_norm(q, layer.gamma_q, c.eps)
        o = shared_kv_attention(q, p, keys, c.tau, c.rope_dims, c.rope_base)
        out[s] = (o, sel, scores)
    return out


def hybrid_decode(layer: LayerState, step: StepInputs, seqs=None):
    decode_update(layer, step)
    return decode_attend(layer, step, seqs)


# ---------------------------------------------------------------------------
# sizing
# ---------------------------------------------------------------------------

def kv_state_bytes(context: int, layers, bytes_per_value: int = 2) -> int:
    """Bytes of KV state of one sequence at `context` tokens.

    layers: iterable of (m, entry_width, window, window_width): a layer keeps
    floor(context/m) entries of entry_width values plus `window` raw rows of
    window_width values.
    """
    total = 0
    for m, entry_width, window, window_width in layers:
        total += (context // m) * entry_width * bytes_per_value
        total += window * window_width * bytes_per_value
    return total
