"""Seeded synthetic inputs in the cache byte layouts of the decode step.

Every array is drawn from numpy's PCG64 with a fixed seed and stored in the
exact byte format the library reads: float32 values, bfloat16 bit patterns
(uint16) or e4m3 codes (uint8) with one float32 scale per row. The float to
bfloat16 / e4m3 casts used to synthesize cache bytes are torch's library
casts; neither the oracle nor the CUDA path uses them.

Workloads (the shapes and value distributions of the benchmark's five
configurations):
  tiny_c4_fp32      C4 layer built end to end from hidden states, fp32, B=1,
                    4096-token prefix, decode at position 4096.
  c128_dense_bf16   dense C128 layer, B=8, 65536-token context, bf16.
  c4_sparse         sparse C4 layer (131072-token context at full size), fp8
                    caches, 5% of entries with 4x-scaled rows.
  compressor_prefill  8 x 4096 new bf16 tokens into a C4 and a C128 compressor.
  stack_1m          two C4 + two C128 layers at 1M context, B=4, 16 steps.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace

import numpy as np
import torch

PAGE_POSITIONS = 256
FP8_GAIN = 112.0          # synthetic e4m3 rows: codes of N(0,1)*112 (clipped), scale 1/112
FP8_LIMIT = 448.0
# synthetic e2m1 rows: magnitude codes 0..7 (values 0 .5 1 1.5 2 3 4 6) with about the frequencies
# of N(0,1)*2 rounded to that grid, scale 1/2 (times the row's gain)
FP4_CODE_PROBS = [0.10, 0.19, 0.18, 0.16, 0.13, 0.14, 0.07, 0.03]
FP4_GAIN = 2.0


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_f32(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    """float32 N(0, std^2) samples, drawn in chunks to bound the float64 peak."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    chunk = 1 << 24
    for a in range(0, n, chunk):
        b = min(n, a + chunk)
        out[a:b] = rng.standard_normal(b - a, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out.reshape(shape)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def fp8_codes(x: np.ndarray) -> np.ndarray:
    x = np.clip(np.ascontiguousarray(x, dtype=np.float32), -FP8_LIMIT, FP8_LIMIT)
    t = torch.from_numpy(x).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def encode_values(x: np.ndarray, dtype: str) -> np.ndarray:
    """Synthetic values -> stored codes of `dtype` (f32 / bf16)."""
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return bf16_bits(x)
    raise ValueError(dtype)


def synth_rows(rng, shape, dtype: str, std: float = 1.0, row_gain=None):
    """Rows [..., D] of a cache in `dtype`, values ~ N(0, std^2) * row_gain.

    Returns (codes, scales) with scales [...] float32 (ones unless fp8).
    """
    x = normal_f32(rng, shape)
    lead = shape[:-1]
    gain = np.ones(lead, dtype=np.float32) if row_gain is None else row_gain.astype(np.float32)
    if dtype == "fp8":
        codes = fp8_codes(x * np.float32(FP8_GAIN))
        scales = (gain * np.float32(std / FP8_GAIN)).astype(np.float32)
        return codes, scales
    if dtype == "fp4":  # e2m1 codes drawn directly (magnitude codes 0..7, random sign), packed
        mag = rng.choice(8, size=shape, p=FP4_CODE_PROBS).astype(np.uint8)
        sign = (rng.random(shape) < 0.5).astype(np.uint8) << 3
        c = mag | sign
        codes = (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)
        scales = (gain * np.float32(std / FP4_GAIN)).astype(np.float32)
        return codes, scales
    x *= np.float32(std)
    x *= gain[..., None]
    return encode_values(x, dtype), np.ones(lead, dtype=np.float32)


# ---------------------------------------------------------------------------
# layer and step containers
# ---------------------------------------------------------------------------

@dataclass
class LayerSpec:
    kind: str                 # "c4" or "c128"
    m: int
    H: int
    D: int
    W: int = 128
    k: int = 512
    H_I: int = 0
    d_I: int = 0
    rope_dims: int = 64
    rope_base: float = 10000.0
    idx_rope_dims: int = 0
    q_idx_rope: bool = False
    eps: float = 1e-6
    cache_dtype: str = "bf16"   # compressed main-KV cache
    swa_dtype: str = "bf16"     # sliding-window ring
    idx_dtype: str = "fp8"      # indexer-key cache
    kv_dtype: str = "bf16"      # new-token kv / gate inputs
    q_dtype: str = "bf16"       # query
    q_idx_dtype: str = "fp8"    # indexer query
    w_dtype: str = "bf16"       # indexer head weights
    out_dtype: str = "bf16"     # f32, bf16 or fp8 (128-channel blocks)
    q_norm: bool = False        # the layer RMS-norms each query head before RoPE

    @property
    def per_page(self) -> int:
        return PAGE_POSITIONS // self.m


@dataclass
class LayerArrays:
    spec: LayerSpec
    B: int
    gamma: np.ndarray            # [D] float32
    pages: np.ndarray            # [num_pages, 256/m, D] codes
    scales: np.ndarray           # [num_pages, 256/m] float32
    block_table: np.ndarray      # [B, max_blocks] int32
    swa_rows: np.ndarray         # [B, W, D] codes
    swa_scales: np.ndarray       # [B, W] float32
    state: np.ndarray            # [B, m, 2D] float32 (kv then gate)
    gamma_idx: np.ndarray | None = None
    idx_pages: np.ndarray | None = None
    idx_scales: np.ndarray | None = None
    idx_block_table: np.ndarray | None = None
    idx_state: np.ndarray | None = None
    gamma_q: np.ndarray | None = None  # [D] float32 query norm weight (q_norm layers)

    @property
    def max_entries(self) -> int:
        return self.block_table.shape[1] * self.spec.per_page

    def copy(self) -> "LayerArrays":
        kw = {}
        for f in self.__dataclass_fields__:
            v = getattr(self, f)
            kw[f] = v.copy() if isinstance(v, np.ndarray) else v
        return LayerArrays(**kw)


@dataclass
class StepArrays:
    pos: np.ndarray              # [B] int32
    kv: np.ndarray               # [B, D] codes (kv_dtype)
    gate: np.ndarray             # [B, D] codes
    q: np.ndarray                # [B, H, D] codes (q_dtype)
    q_idx: np.ndarray | None = None        # [B, H_I, d_I] codes (q_idx_dtype)
    q_idx_scale: np.ndarray | None = None  # [B, H_I] float32
    w: np.ndarray | None = None            # [B, H_I] codes (w_dtype)
    idx_kv: np.ndarray | None = None       # [B, d_I] codes (kv_dtype)
    idx_gate: np.ndarray | None = None


def block_table(rng, B: int, blocks_per_seq: int, spare_pages: int = 0) -> tuple[np.ndarray, int]:
    """A random one-to-one map (sequence, logical block) -> physical page."""
    num_pages = B * blocks_per_seq + spare_pages
    perm = rng.permutation(num_pages).astype(np.int32)
    return perm[: B * blocks_per_seq].reshape(B, blocks_per_seq).copy(), num_pages


def make_layer(spec: LayerSpec, B: int, context_entries: int, seed: int, *,
               value_std: float = 1.0, outlier_frac: float = 0.0, outlier_gain: float = 4.0,
               spare_blocks: int = 2, spare_pages: int = 3) -> LayerArrays:
    """A layer whose caches already hold `context_entries` entries per sequence.

    Every physical row (used or not) is filled with random values so that a
    read outside the visible range changes the result. The outlier rows (a
    Bernoulli(outlier_frac) subset of physical rows) are scaled by
    outlier_gain in both the main cache and the indexer-key cache.
    """
    rng = rng_for(seed)
    per_page = spec.per_page
    blocks = -(-max(context_entries, 1) // per_page) + spare_blocks
    bt, num_pages = block_table(rng, B, blocks, spare_pages)
    gain = np.ones((num_pages, per_page), dtype=np.float32)
    if outlier_frac > 0:
        mask = rng.random((num_pages, per_page)) < outlier_frac
        gain[mask] = np.float32(outlier_gain)
    pages, scales = synth_rows(rng, (num_pages, per_page, spec.D), spec.cache_dtype,
                               value_std, gain)
    swa_rows, swa_scales = synth_rows(rng, (B, spec.W, spec.D), spec.swa_dtype, value_std)
    state = normal_f32(rng, (B, spec.m, 2 * spec.D))
    if spec.kv_dtype == "bf16":  # the ring holds float32 copies of bf16 inputs
        state = (bf16_bits(state).astype(np.uint32) << 16).view(np.float32)
    la = LayerArrays(spec=spec, B=B, gamma=np.ones(spec.D, dtype=np.float32), pages=pages,
                     scales=scales, block_table=bt, swa_rows=swa_rows, swa_scales=swa_scales,
                     state=state)
    if spec.q_norm:
        la.gamma_q = (1.0 + 0.1 * normal_f32(rng, (spec.D,))).astype(np.float32)
    if spec.kind == "c4":
        la.gamma_idx = np.ones(spec.d_I, dtype=np.float32)
        la.idx_pages, la.idx_scales = synth_rows(rng, (num_pages, per_page, spec.d_I),
                                                 spec.idx_dtype, 1.0, gain)
        la.idx_block_table = bt
        st = normal_f32(rng, (B, spec.m, 2 * spec.d_I))
        if spec.kv_dtype == "bf16":
            st = (bf16_bits(st).astype(np.uint32) << 16).view(np.float32)
        la.idx_state = st
    return la


def make_step(spec: LayerSpec, B: int, pos, seed: int, *, q_std: float = 1.0,
              kv_std: float = 1.0) -> StepArrays:
    """Inputs of one decode step: the new token's kv/gate, q, and indexer inputs."""
    rng = rng_for(seed)
    pos = np.broadcast_to(np.asarray(pos, dtype=np.int32), (B,)).copy()
    st = StepArrays(pos=pos,
                    kv=encode_values(normal_f32(rng, (B, spec.D), kv_std), spec.kv_dtype),
                    gate=encode_values(normal_f32(rng, (B, spec.D)), spec.kv_dtype),
                    q=encode_values(normal_f32(rng, (B, spec.H, spec.D), q_std), spec.q_dtype))
    if spec.kind == "c4":
        if spec.q_idx_dtype == "fp8":
            st.q_idx = fp8_codes(normal_f32(rng, (B, spec.H_I, spec.d_I)) * np.float32(FP8_GAIN))
            st.q_idx_scale = np.full((B, spec.H_I), 1.0 / FP8_GAIN, dtype=np.float32)
        else:
            st.q_idx = encode_values(normal_f32(rng, (B, spec.H_I, spec.d_I)), spec.q_idx_dtype)
            st.q_idx_scale = np.ones((B, spec.H_I), dtype=np.float32)
        st.w = encode_values(normal_f32(rng, (B, spec.H_I)), spec.w_dtype)
        st.idx_kv = encode_values(normal_f32(rng, (B, spec.d_I)), spec.kv_dtype)
        st.idx_gate = encode_values(normal_f32(rng, (B, spec.d_I)), spec.kv_dtype)
    return st


# ---------------------------------------------------------------------------
# the five workloads
# ---------------------------------------------------------------------------

TINY_SPEC = LayerSpec(kind="c4", m=4, H=16, D=128, W=128, k=64, H_I=4, d_I=32, rope_dims=64,
                      idx_rope_dims=16, q_idx_rope=True, cache_dtype="f32", swa_dtype="f32",
                      idx_dtype="f32", kv_dtype="f32", q_dtype="f32", q_idx_dtype="f32",
                      w_dtype="f32", out_dtype="f32")


@dataclass
class TinyWorkload:
    layer: LayerArrays           # empty caches, to be built from the prefix
    prefix_kv: np.ndarray        # [L, D] float32
    prefix_gate: np.ndarray
    prefix_idx_kv: np.ndarray    # [L, d_I]
    prefix_idx_gate: np.ndarray
    step: StepArrays             # decode at position L


def tiny_c4_fp32(seed: int = 0, context: int = 4096, hidden: int = 256) -> TinyWorkload:
    """C4 decode built end to end from hidden states ~ N(0,1) with projections
    W ~ N(0, 1/hidden); the projections are the model's linear maps, done here
    in float64 and rounded to float32 (they are inputs to the decode step)."""
    spec = TINY_SPEC
    rng = rng_for(seed)
    T = context + 1
    h = rng.standard_normal((T, hidden))
    sd = 1.0 / np.sqrt(hidden)

    def proj(rows):
        return rng.standard_normal((rows, hidden)) * sd

    W_kv, W_g = proj(spec.D), proj(spec.D)
    W_kvI, W_gI = proj(spec.d_I), proj(spec.d_I)
    W_q, W_qI, W_w = proj(spec.H * spec.D), proj(spec.H_I * spec.d_I), proj(spec.H_I)
    f = lambda a: np.ascontiguousarray(a, dtype=np.float32)  # noqa: E731
    kv, gate = f(h @ W_kv.T), f(h @ W_g.T)
    ikv, igate = f(h @ W_kvI.T), f(h @ W_gI.T)
    hp = h[context]
    n_entries = context // spec.m + 1
    blocks = -(-n_entries // spec.per_page) + 1
    bt, num_pages = block_table(rng, 1, blocks, 5)
    junk = lambda *s: normal_f32(rng, s)  # noqa: E731  unwritten rows hold junk
    layer = LayerArrays(
        spec=spec, B=1,
        gamma=f(1.0 + 0.1 * rng.standard_normal(spec.D)),
        pages=junk(num_pages, spec.per_page, spec.D), scales=np.ones((num_pages, spec.per_page), np.float32),
        block_table=bt,
        swa_rows=junk(1, spec.W, spec.D), swa_scales=np.ones((1, spec.W), np.float32),
        state=junk(1, spec.m, 2 * spec.D),
        gamma_idx=f(1.0 + 0.1 * rng.standard_normal(spec.d_I)),
        idx_pages=junk(num_pages, spec.per_page, spec.d_I),
        idx_scales=np.ones((num_pages, spec.per_page), np.float32),
        idx_block_table=bt.copy(),
        idx_state=junk(1, spec.m, 2 * spec.d_I))
    step = StepArrays(pos=np.array([context], dtype=np.int32), kv=kv[context:context + 1].copy(),
                      gate=gate[context:context + 1].copy(),
                      q=f((W_q @ hp).reshape(1, spec.H, spec.D)),
                      q_idx=f((W_qI @ hp).reshape(1, spec.H_I, spec.d_I)),
                      q_idx_scale=np.ones((1, spec.H_I), np.float32),
                      w=f((W_w @ hp).reshape(1, spec.H_I)),
                      idx_kv=ikv[context:context + 1].copy(), idx_gate=igate[context:context + 1].copy())
    return TinyWorkload(layer=layer, prefix_kv=kv[:context].copy(), prefix_gate=gate[:context].copy(),
                        prefix_idx_kv=ikv[:context].copy(), prefix_idx_gate=igate[:context].copy(),
                        step=step)


C128_SPEC = LayerSpec(kind="c128", m=128, H=64, D=512, W=128, k=0, cache_dtype="bf16",
                      swa_dtype="bf16", kv_dtype="bf16", q_dtype="bf16", out_dtype="bf16")

C4_SPEC = LayerSpec(kind="c4", m=4, H=64, D=512, W=128, k=512, H_I=64, d_I=128,
                    idx_rope_dims=64, cache_dtype="fp8", swa_dtype="fp8", idx_dtype="fp8",
                    kv_dtype="bf16", q_dtype="bf16", q_idx_dtype="fp8", w_dtype="bf16",
                    out_dtype="bf16")
# the same layer with an fp4 (e2m1) indexer-key cache
C4_FP4_SPEC = replace(C4_SPEC, idx_dtype="fp4")


def c128_dense_bf16(seed: int = 1, B: int = 8, context: int = 65536, steps: int = 1):
    """Dense C128 layer: entries, window rows and queries ~ N(0,1)/sqrt(512)."""
    spec = C128_SPEC
    std = 1.0 / np.sqrt(spec.D)
    layer = make_layer(spec, B, context // spec.m, seed, value_std=std)
    st = [make_step(spec, B, context + i, seed * 1000 + 17 + i, q_std=std) for i in range(steps)]
    return layer, st


def c4_sparse(seed: int = 2, B: int = 32, context: int = 131072, steps: int = 1,
              outlier_frac: float = 0.05, spec: LayerSpec = C4_SPEC):
    """Sparse C4 layer with fp8 caches; entries ~ N(0,1), 5% of rows x4."""
    layer = make_layer(spec, B, context // spec.m, seed, outlier_frac=outlier_frac)
    st = [make_step(spec, B, context + i, seed * 1000 + 17 + i) for i in range(steps)]
    return layer, st


@dataclass
class PrefillWorkload:
    cu_seqlens: np.ndarray   # [B+1] int32
    start_pos: np.ndarray    # [B] int32
    kv4: np.ndarray          # [T, D] bf16 bits: inputs of the C4 compressor
    gate4: np.ndarray
    kv128: np.ndarray        # inputs of the C128 compressor
    gate128: np.ndarray
    layer4: LayerArrays      # C4 caches + state
    layer128: LayerArrays


def compressor_prefill(seed: int = 3, B: int = 8, tokens_per_seq: int = 4096, D: int = 512,
                       start_pos=None, cache_dtype: str = "bf16") -> PrefillWorkload:
    """New tokens for two compressors (m = 4 and m = 128), bf16 inputs ~ N(0,1)
    (the projected hidden states), written into paged caches."""
    rng = rng_for(seed)
    T = B * tokens_per_seq
    cu = (np.arange(B + 1) * tokens_per_seq).astype(np.int32)
    sp = np.zeros(B, np.int32) if start_pos is None else np.asarray(start_pos, np.int32)
    kv4, g4 = bf16_bits(normal_f32(rng, (T, D))), bf16_bits(normal_f32(rng, (T, D)))
    kv128, g128 = bf16_bits(normal_f32(rng, (T, D))), bf16_bits(normal_f32(rng, (T, D)))
    layers = []
    for m in (4, 128):
        spec = LayerSpec(kind="c128", m=m, H=64, D=D, cache_dtype=cache_dtype, swa_dtype="bf16")
        ctx = int(sp.max()) + tokens_per_seq
        la = make_layer(spec, B, ctx // m + 1, seed * 100 + m, spare_blocks=1)
        layers.append(la)
    return PrefillWorkload(cu, sp, kv4, g4, kv128, g128, layers[0], layers[1])


@dataclass
class ProjectionWorkload:
    cu_seqlens: np.ndarray   # [B+1] int32
    start_pos: np.ndarray    # [B] int32
    hidden: np.ndarray       # [T, Hd] bf16 bits, ~ N(0, 1)
    w4: np.ndarray           # [2D, Hd] bf16 bits, ~ N(0, 1/Hd): the C4 compressor's kv rows, then gate rows
    w128: np.ndarray         # the C128 compressor's
    layer4: LayerArrays      # C4 caches + state
    layer128: LayerArrays


def projection_prefill(seed: int = 5, B: int = 8, tokens_per_seq: int = 4096, hidden_dim: int = 4096,
                       D: int = 512, start_pos=None, lens=None, cache_dtype: str = "bf16") -> ProjectionWorkload:
    """Hidden states of new tokens and the projection weights of two compressors (m = 4 and
    m = 128): hidden ~ N(0,1), weights ~ N(0, 1/hidden_dim), so kv and gate come out ~ N(0,1)
    like the compressor prefill's inputs. `lens` (per sequence) overrides tokens_per_seq."""
    rng = rng_for(seed)
    lens = np.full(B, tokens_per_seq, np.int64) if lens is None else np.asarray(lens, np.int64)
    B = lens.shape[0]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    sp = np.zeros(B, np.int32) if start_pos is None else np.asarray(start_pos, np.int32)
    hidden = bf16_bits(normal_f32(rng, (T, hidden_dim)))
    w4 = bf16_bits(normal_f32(rng, (2 * D, hidden_dim), 1.0 / np.sqrt(hidden_dim)))
    w128 = bf16_bits(normal_f32(rng, (2 * D, hidden_dim), 1.0 / np.sqrt(hidden_dim)))
    layers = []
    for m in (4, 128):
        spec = LayerSpec(kind="c128", m=m, H=64, D=D, cache_dtype=cache_dtype, swa_dtype="bf16")
        ctx = int((sp + lens).max())
        la = make_layer(spec, B, ctx // m + 1, seed * 100 + m, spare_blocks=1)
        layers.append(la)
    return ProjectionWorkload(cu, sp, hidden, w4, w128, layers[0], layers[1])


def stack_1m(seed: int = 4, B: int = 4, context: int = 1 << 20, steps: int = 16):
    """Two C4 (fp8) and two C128 (bf16) layers at 1M context; per-layer inputs
    for `steps` consecutive decode steps."""
    layers, step_sets = [], []
    for li, spec in enumerate((C4_SPEC, C128_SPEC, C4_SPEC, C128_SPEC)):
        la = make_layer(spec, B, context // spec.m, seed * 10 + li)
        layers.append(la)
        step_sets.append([make_step(spec, B, context + i, seed * 10000 + li * 100 + i)
                          for i in range(steps)])
    return layers, step_sets
