"""Wrap the synthetic workloads' byte arrays into the oracle's containers.

Test infrastructure. Inputs are decoded exactly (bfloat16 bits, e4m3 codes
times their float32 scale) with the oracle's own codecs; caches are deep
copies, so the oracle updates its own state and never the caller's arrays.
"""

from __future__ import annotations

import numpy as np

from . import dsv4_oracle as O


def decode_input(codes, dtype: str, scales=None) -> np.ndarray:
    if codes is None:
        return None
    if dtype == "f32":
        return np.asarray(codes, np.float32).astype(np.float64)
    if dtype == "bf16":
        return O.bf16_decode(codes)
    if dtype == "fp8":
        return O.e4m3_decode(codes) * np.asarray(scales, np.float32).astype(np.float64)[..., None]
    if dtype == "fp4":
        return O.decode_rows(codes, scales, "fp4")
    raise ValueError(dtype)


def layer_config(spec) -> O.LayerConfig:
    return O.LayerConfig(kind=spec.kind, m=spec.m, H=spec.H, D=spec.D, W=spec.W, k=spec.k,
                         H_I=spec.H_I, d_I=spec.d_I, rope_dims=spec.rope_dims,
                         rope_base=spec.rope_base, idx_rope_dims=spec.idx_rope_dims,
                         q_idx_rope=spec.q_idx_rope, eps=spec.eps)


def layer_state(la) -> O.LayerState:
    spec = la.spec
    cfg = layer_config(spec)
    st = O.LayerState(
        cfg=cfg, gamma=la.gamma.astype(np.float64),
        main_state=O.CompressorState(spec.m, spec.D, spec.D, la.state.copy()),
        main_cache=O.PagedCache(spec.cache_dtype, spec.m, spec.D, la.pages.copy(),
                                la.scales.copy(), la.block_table.copy()),
        window=O.WindowRing(spec.swa_dtype, spec.W, spec.D, la.swa_rows.copy(),
                            la.swa_scales.copy()))
    if getattr(la, "gamma_q", None) is not None:
        st.gamma_q = la.gamma_q.astype(np.float64)
    if spec.kind == "c4":
        st.gamma_idx = la.gamma_idx.astype(np.float64)
        st.idx_state = O.CompressorState(spec.m, spec.d_I, spec.d_I, la.idx_state.copy())
        st.idx_cache = O.PagedCache(spec.idx_dtype, spec.m, spec.d_I, la.idx_pages.copy(),
                                    la.idx_scales.copy(), la.idx_block_table.copy())
    return st


def step_inputs(spec, st) -> O.StepInputs:
    kvd = spec.kv_dtype
    return O.StepInputs(
        pos=np.asarray(st.pos, np.int64),
        kv=decode_input(st.kv, kvd), gate=decode_input(st.gate, kvd),
        q=decode_input(st.q, spec.q_dtype),
        q_idx=decode_input(st.q_idx, spec.q_idx_dtype, st.q_idx_scale),
        w=decode_input(st.w, spec.w_dtype),
        idx_kv=decode_input(st.idx_kv, kvd), idx_gate=decode_input(st.idx_gate, kvd))
