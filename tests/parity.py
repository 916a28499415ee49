"""Comparison rules shared by the GPU parity tests.

Thresholds (fixed by the problem statement of the method):
  - top-k index sets are bit-exact, except that an index in the symmetric
    difference must have an oracle score within 1e-6 * |s_k| of the oracle's
    k-th score s_k (a near tie);
  - attention outputs: max-abs <= 1e-3 for fp32, and max-abs <= 2e-2 with
    rel-L2 <= 1e-2 for bf16 / fp8 inputs.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

TIE_REL = 1e-6
F32_MAX_ABS = 1e-3
LOWP_MAX_ABS = 2e-2
LOWP_REL_L2 = 1e-2


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import compressed_sparse_kv_dsv4_b200 as dsv4  # noqa: F401  raises if the library is missing
    dsv4.load()


def check_topk(gpu_idx, scores, k: int, n_c: int, ctx: str = "", allow_extra=None):
    """gpu_idx: [k] int (-1 padded); scores: oracle float64 scores of the n_c entries.

    Returns the number of near-tie swaps. `allow_extra` is a set of entry indices
    whose scores may legitimately differ between the two sides (entries the two
    sides built themselves); a swap involving one of them is counted, not failed.
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
    if allow_extra:
        bad = [j for j in bad if j not in allow_extra]
    assert not bad, (f"{ctx}: {len(bad)} indices differ beyond the tie band, e.g. "
                     f"{[(j, s[j], sk) for j in bad[:4]]}")
    return len(diff) // 2


def input_class(spec) -> str:
    """Tolerance class of a layer: fp32 inputs, or bf16 / fp8 inputs."""
    return "f32" if spec.cache_dtype == "f32" else "lowp"


def check_output(got, want, inputs: str, ctx: str = "", stored_bf16: bool = False):
    """inputs: "f32" or "lowp" (bf16 / fp8 inputs). stored_bf16: the output was stored as
    bf16 (8 significant bits), whose round-to-nearest moves a value x by up to half an ulp,
    2^(floor(log2|x|) - 8) <= 2^-8 |x|; that allowance, taken at |want| + the max-abs bound
    (x is the unrounded result, within that bound of want), is added, nothing else."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, f"{ctx}: shape {got.shape} vs {want.shape}"
    assert np.all(np.isfinite(got)), f"{ctx}: non-finite output"
    err = np.abs(got - want)
    bound = F32_MAX_ABS if inputs == "f32" else LOWP_MAX_ABS
    store = 2.0 ** -8 * (np.abs(want) + bound) if stored_bf16 else 0.0
    if inputs == "f32":
        assert np.all(err <= F32_MAX_ABS + store), f"{ctx}: max-abs {err.max():.3e} > {F32_MAX_ABS}"
        return err.max(), None
    rel = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    assert np.all(err <= LOWP_MAX_ABS + store), f"{ctx}: max-abs {err.max():.3e} > {LOWP_MAX_ABS} (+ storage)"
    assert rel <= LOWP_REL_L2, f"{ctx}: rel-L2 {rel:.3e} > {LOWP_REL_L2}"
    return err.max(), rel


def decode_out(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
