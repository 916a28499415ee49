"""Comparison rules shared by the GPU parity tests.

Thresholds (fixed by the problem statement of the method):
  - top-k index sets are bit-exact, except that an index in the symmetric
    difference must have an oracle score within 1e-6 * |s_k| of the oracle's
    k-th score s_k (a near tie);
  - attention outputs: max-abs <= 1e-3 for fp32 inputs, and max-abs <= 2e-2
    with rel-L2 <= 1e-2 for bf16 / fp8 inputs.

Outputs stored as float32 are held to those bounds as written. An output stored
as bf16 is compared with the oracle's output rounded to bf16 by the same rule
(round to nearest even); the bound then grows by one bf16 ulp of that rounded
value, because two values within the bound of each other can round to
neighbouring bf16 numbers.

Rows the decode step writes (window slot, appended compressed and indexer
entries) are rounded into their cache dtype by each side from float32 values
that may differ in the last bit, so a code can sit one rounding step from the
oracle's. `codes_close` states that bound; `row_bytes_equal` says whether the
two sides stored the very same bytes. A top-k swap is excused only for an
appended entry whose stored bytes differ between the sides (the comparison
rule for paths where each side's own compressor feeds its indexer).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle.dsv4_oracle as O

TIE_REL = 1e-6
F32_MAX_ABS = 1e-3
LOWP_MAX_ABS = 2e-2
LOWP_REL_L2 = 1e-2


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import compressed_sparse_kv_dsv4_b200 as dsv4  # noqa: F401  raises if the library is missing
    dsv4.load()


def check_topk(gpu_idx, scores, k: int, n_c: int, ctx: str = "", excused=None):
    """gpu_idx: [k] int (-1 padded); scores: oracle float64 scores of the n_c entries.

    Returns the number of near-tie swaps. `excused` is a set of entry indices whose
    stored key bytes were shown to differ between the two sides (see the module
    docstring); a swap involving one of them is counted, not failed.
    """
    gpu_idx = np.asarray(gpu_idx, dtype=np.int64)
    valid = gpu_idx[gpu_idx >= 0]
    want_n = min(k, n_c)
    assert valid.shape[0] == want_n, f"{ctx}: {valid.shape[0]} valid indices, want {want_n}"
    assert np.all(gpu_idx[want_n:] == -1), f"{ctx}: padding must follow the valid indices"
    assert np.unique(valid).shape[0] == valid.shape[0], f"{ctx}: duplicate indices"
    assert valid.max(initial=-1) < n_c, f"{ctx}: index out of range"
    if n_c <= k:
        assert set(valid.tolist()) == set(range(n_c)), f"{ctx}: n_c <= k must take every entry"
        return 0
    s = np.asarray(scores, dtype=np.float64)
    order = np.lexsort((np.arange(n_c), -s))
    ref = set(order[:k].tolist())
    sk = s[order[k - 1]]
    diff = ref.symmetric_difference(set(valid.tolist()))
    bad = [j for j in diff if abs(s[j] - sk) > TIE_REL * abs(sk)]
    if excused:
        bad = [j for j in bad if j not in excused]
    assert not bad, (f"{ctx}: {len(bad)} indices differ beyond the tie band, e.g. "
                     f"{[(j, s[j], sk) for j in bad[:4]]}")
    return len(diff) // 2


def input_class(spec) -> str:
    """Tolerance class of a layer: fp32 inputs, or bf16 / fp8 inputs."""
    return "f32" if spec.cache_dtype == "f32" else "lowp"


def bf16_round(x) -> np.ndarray:
    """float64 -> the nearest bf16 value (via float32, ties to even), as float64."""
    return O.bf16_decode(O.bf16_encode(np.asarray(x, dtype=np.float64).astype(np.float32)))


def bf16_ulp(v) -> np.ndarray:
    """Spacing of bf16 numbers at |v| (8 significant bits): 2^(floor(log2|v|) - 7)."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 7)


def check_output(got, want, inputs: str, ctx: str = "", out_dtype: str = "f32"):
    """inputs: "f32" or "lowp" (bf16 / fp8 inputs); out_dtype: how `got` was stored.

    A float32 output is held to the bounds as written. A bf16 output is compared with
    bf16(want), within the bound plus one bf16 ulp of bf16(want)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, f"{ctx}: shape {got.shape} vs {want.shape}"
    assert np.all(np.isfinite(got)), f"{ctx}: non-finite output"
    bound = F32_MAX_ABS if inputs == "f32" else LOWP_MAX_ABS
    if out_dtype == "bf16":
        want = bf16_round(want)
        limit = bound + bf16_ulp(want)
    elif out_dtype == "f32":
        limit = bound
    else:
        raise ValueError(out_dtype)
    err = np.abs(got - want)
    assert np.all(err <= limit), f"{ctx}: max-abs {err.max():.3e} > {bound} ({out_dtype} output)"
    if inputs == "f32":
        return err.max(), None
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert rel <= LOWP_REL_L2, f"{ctx}: rel-L2 {rel:.3e} > {LOWP_REL_L2}"
    return err.max(), rel


def e4m3_step(v, scale) -> np.ndarray:
    """Spacing of the e4m3 grid (times `scale`) at |v|: 2^(floor(log2(|v|/scale)) - 3) for
    normal codes, 2^-9 below 2^-6 (the subnormal spacing)."""
    a = np.abs(np.asarray(v, np.float64)) / np.asarray(scale, np.float64)
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -6)))
    return np.exp2(e - 3) * np.asarray(scale, np.float64)


def check_output_fp8(codes, scales, want, inputs: str, ctx: str = ""):
    """An fp8 output (e4m3 codes [H, D] with one scale per 128-channel block, R22) against the
    oracle's output rounded the same way (its own block scales): within the bound plus one
    e4m3 step of the rounded value, and rel-L2 within the bound."""
    codes = np.asarray(codes, np.uint8)
    scales = np.asarray(scales, np.float32)
    H, D = codes.shape
    blk = O.OUT_BLOCK
    got = O.e4m3_decode(codes) * np.repeat(scales.astype(np.float64), blk, axis=1)
    _, wsc, want_q = O.store_output(np.asarray(want, np.float64), "fp8")
    step = e4m3_step(want_q, np.repeat(wsc.astype(np.float64), blk, axis=1))
    bound = F32_MAX_ABS if inputs == "f32" else LOWP_MAX_ABS
    err = np.abs(got - want_q)
    assert np.all(np.isfinite(got)), f"{ctx}: non-finite output"
    assert np.all(err <= bound + step), f"{ctx}: max-abs {err.max():.3e} > {bound} (+ one e4m3 step)"
    assert np.all(np.abs(scales.astype(np.float64) - wsc) <= 2e-2 * wsc), f"{ctx}: block scales"
    rel = np.linalg.norm(got - want_q) / max(np.linalg.norm(want_q), 1e-30)
    assert rel <= LOWP_REL_L2, f"{ctx}: rel-L2 {rel:.3e} > {LOWP_REL_L2}"
    return err.max(), rel


def decode_out(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def codes_close(gpu_codes, ref_codes, gpu_scales, ref_scales, dtype, ctx, max_frac: float = 0.01):
    """Rows rounded into a cache dtype by the two sides from float32 values that may
    differ in the last bits: equal, or one rounding step apart (and few of them).

    The GPU pools a block of up to m = 128 tokens with float32 sums, whose absolute error
    reaches about m * 2^-24 of the row's largest value; an element much smaller than that
    can therefore round to a different bf16 value. The bf16 bound is one bf16 step of the
    element plus 2^-16 of the row's largest magnitude."""
    if dtype == "f32":
        g = np.asarray(gpu_codes, np.float64)
        r = np.asarray(ref_codes, np.float64)
        assert np.max(np.abs(g - r)) <= 2e-5 * max(1.0, np.max(np.abs(r))), ctx
        return
    if dtype == "bf16":
        g, r = O.bf16_decode(gpu_codes), O.bf16_decode(ref_codes)
        floor = 2.0 ** -16 * np.max(np.abs(r), initial=0.0)
        assert np.all(np.abs(g - r) <= 2.0 ** -7 * np.abs(r) + floor + 1e-30), ctx
        return
    gs, rs = np.asarray(gpu_scales, np.float64), np.asarray(ref_scales, np.float64)
    assert np.all(np.abs(gs - rs) <= 1e-6 * rs), f"{ctx}: scales"
    if dtype == "fp4":  # e2m1 codes two per byte: sign bit 3, magnitude codes 0..7 in value order
        g = O.fp4_unpack(np.asarray(gpu_codes)).astype(np.int32)
        r = O.fp4_unpack(np.asarray(ref_codes)).astype(np.int32)
        same_sign = (g & 0x8) == (r & 0x8)
        step = np.abs((g & 0x7) - (r & 0x7))
        zero = ((g & 0x7) == 0) & ((r & 0x7) <= 1) | ((r & 0x7) == 0) & ((g & 0x7) <= 1)
        assert np.all((same_sign & (step <= 1)) | zero), f"{ctx}: fp4 codes more than one step apart"
        assert np.mean(g != r) <= max_frac, f"{ctx}: too many fp4 rounding differences"
        return
    g = np.asarray(gpu_codes).astype(np.int32)
    r = np.asarray(ref_codes).astype(np.int32)
    same_sign = (g & 0x80) == (r & 0x80)
    step = np.abs((g & 0x7F) - (r & 0x7F))
    zero = ((g & 0x7F) == 0) & ((r & 0x7F) <= 1) | ((r & 0x7F) == 0) & ((g & 0x7F) <= 1)
    ok = (same_sign & (step <= 1)) | zero
    assert np.all(ok), f"{ctx}: fp8 codes more than one step apart"
    assert np.mean(g != r) <= max_frac, f"{ctx}: too many fp8 rounding differences"


def row_bytes_equal(gpu_codes, ref_codes, gpu_scale, ref_scale) -> bool:
    """The two sides stored the same code bytes and the same float32 scale."""
    g = np.ascontiguousarray(gpu_codes)
    r = np.ascontiguousarray(ref_codes)
    if g.dtype == np.float32 or r.dtype == np.float32:
        g, r = g.astype(np.float32).view(np.uint32), r.astype(np.float32).view(np.uint32)
    return bool(np.array_equal(g, r)) and np.float32(gpu_scale) == np.float32(ref_scale)


def check_step_writes(dl, ol, spec, st):
    """Every row a decode step wrote, read back from the device layer `dl` and compared
    with the oracle layer `ol` after both ran the step: the window row of each sequence's
    position, both compressor state rings (exact: they hold the inputs), and each entry the
    step completed in the main and (C4) indexer caches. Returns {seq: set of appended
    entries whose stored bytes differ between the two sides}."""
    import compressed_sparse_kv_dsv4_b200 as dsv4

    differ = {}
    ring_rows = dsv4.to_numpy_codes(dl.ring.rows, spec.swa_dtype)
    ring_sc = dl.ring.scales.cpu().numpy()
    assert np.array_equal(dl.state.buf.cpu().numpy(), ol.main_state.buf), "main compressor state"
    if spec.kind == "c4":
        assert np.array_equal(dl.idx_state.buf.cpu().numpy(), ol.idx_state.buf), "indexer compressor state"
    for s in range(np.asarray(st.pos).shape[0]):
        p = int(st.pos[s])
        slot = p % spec.W
        codes_close(ring_rows[s, slot], ol.window.rows[s, slot], ring_sc[s, slot], ol.window.scales[s, slot],
                    spec.swa_dtype, f"seq {s}: window row of position {p}", max_frac=0.05)
        differ[s] = set()
        for j in range(p // spec.m, (p + 1) // spec.m):  # the entry this step completed, if any
            caches = [(dl.cache, ol.main_cache, spec.cache_dtype, "main")]
            if spec.kind == "c4":
                caches.append((dl.idx_cache, ol.idx_cache, spec.idx_dtype, "indexer"))
            for dc, oc, dt, name in caches:
                pg, sl = oc.locate(s, j)
                codes = dsv4.to_numpy_codes(dc.pages[int(pg), int(sl)], dt)
                sc = float(dc.scales[int(pg), int(sl)].item())
                codes_close(codes, oc.pages[pg, sl], sc, oc.scales[pg, sl], dt,
                            f"seq {s}: appended {name} entry {j}", max_frac=0.05)
                if not row_bytes_equal(codes, oc.pages[pg, sl], sc, oc.scales[pg, sl]):
                    differ[s].add(j)
    return differ
