"""GPU parity of dsv4_compress_project (the compressor with its input projection in front)
against the oracle's projection (each output rounded once to bf16 from the exact product)
followed by the oracle's compressor.

The GPU accumulates the hidden-dim products in fp32 on the tensor cores, so an output whose
exact value lies within the fp32 sum's error of a bf16 rounding midpoint may round to the
neighbouring bf16 value: projected values are compared within one bf16 step, and only a
small fraction may differ at all. The compressor then runs on the two sides' own projected
inputs, so its cache rows are compared as end-to-end results (decoded values within one
step of the cache dtype plus the movement such input differences cause) and its state ring
(the tail tokens' kv and gate) within one bf16 step.
"""

import numpy as np
import pytest
import torch

import compressed_sparse_kv_dsv4_b200 as dsv4
import oracle.dsv4_oracle as O
import synthetic as W
from oracle import adapters as OA
from tests.parity import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _bf16_close(gpu_bits, ref_bits, err, ctx, max_frac=0.01):
    """Projected values: the GPU's fp32 sum is within `err` (per element) of the exact one, so
    its bf16 rounding is within one bf16 step of |r| + err of the oracle's, plus err."""
    if np.asarray(ref_bits).size == 0:
        return 0.0
    g = O.bf16_decode(np.asarray(gpu_bits).view(np.uint16))
    r = O.bf16_decode(np.asarray(ref_bits).view(np.uint16))
    step = np.exp2(np.floor(np.log2(np.maximum(np.abs(r) + err, 2.0 ** -126))) - 7)
    assert np.all(np.abs(g - r) <= step + err), f"{ctx}: more than one bf16 step apart"
    frac = np.mean(g != r)
    assert frac <= max_frac, f"{ctx}: {frac:.4f} of the values differ"
    return frac


def _sum_error_bound(h, w):
    """Bound on |fp32 sum - exact| of every output of h [T, K] . w [N, K]^T: recursive fp32
    summation of K exact products errs by at most K 2^-24 sum_i |h_i w_i|; twice that covers
    the tensor core's own order of additions."""
    K = h.shape[1]
    return 2.0 * K * 2.0 ** -24 * (np.abs(h) @ np.abs(w).T)


def _rows_close_e2e(g_codes, g_scale, r_codes, r_scale, dtype, ctx):
    """A cache row each side built from its own projected inputs, which may differ by one
    bf16 step in a few values. A changed kv or gate value moves its channel's pooled value by
    up to a few 2^-8 of the channel's inputs (through the value, and through the softmax
    weights), and the RMSNorm scales that by 1/rms: every decoded value agrees within one
    rounding step of the cache dtype plus 2^-6 of itself plus 2^-3 of the row's rms, and at most
    10 % of them (the channels a changed input reached) need more than the first two terms.
    An fp8 or fp4 row's scale (amax/448, amax/6) agrees within 2^-5."""
    g = O.decode_rows(np.asarray(g_codes)[None], np.array([g_scale], np.float32), dtype)[0]
    r = O.decode_rows(np.asarray(r_codes)[None], np.array([r_scale], np.float32), dtype)[0]
    if dtype == "fp8":
        assert abs(float(g_scale) - float(r_scale)) <= 2.0 ** -5 * float(r_scale), f"{ctx}: scale"
        step = np.exp2(np.floor(np.log2(np.maximum(np.abs(r) / float(r_scale), 2.0 ** -6))) - 3) * float(r_scale)
    elif dtype == "fp4":  # e2m1 magnitudes 0 .5 1 1.5 2 3 4 6: steps of 1/2, 1, 2 (times the scale)
        assert abs(float(g_scale) - float(r_scale)) <= 2.0 ** -5 * float(r_scale), f"{ctx}: scale"
        a = np.abs(r) / float(r_scale)
        step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0)) * float(r_scale)
    else:
        step = np.exp2(np.floor(np.log2(np.maximum(np.abs(r), 2.0 ** -126))) - 7)
    rms = float(np.sqrt(np.mean(r * r)))
    tight = step + 2.0 ** -6 * np.abs(r)
    d = np.abs(g - r)
    assert np.all(d <= tight + 2.0 ** -3 * rms), f"{ctx}: values"
    assert np.mean(d > tight) <= 0.10, f"{ctx}: {np.mean(d > tight):.3f} of the values moved"


def _run(wl, which, seqs=None):
    """GPU projection + compressor for compressor `which` (4 or 128); oracle on `seqs`."""
    la = wl.layer4 if which == 4 else wl.layer128
    w = wl.w4 if which == 4 else wl.w128
    spec = la.spec
    D = spec.D
    dl = dsv4.DeviceLayer.from_arrays(la)
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()  # noqa: E731
    hid = dsv4.to_device_codes(wl.hidden, "bf16", "cuda")
    wd = dsv4.to_device_codes(w, "bf16", "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    kv, gate = dsv4.compress_project(hid, wd, f(wl.cu_seqlens), f(wl.start_pos), dl.state, dl.cache, dl.gamma,
                                     eps=1e-6, rope_dims=64, rope_base=1e4, d_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    gkv = dsv4.to_numpy_codes(kv, "bf16").view(np.uint16)
    ggate = dsv4.to_numpy_codes(gate, "bf16").view(np.uint16)
    ol = OA.layer_state(la)
    seqs = range(len(wl.cu_seqlens) - 1) if seqs is None else seqs
    w_v = O.bf16_decode(w)
    pages = dsv4.to_numpy_codes(dl.cache.pages, spec.cache_dtype)
    scales = dl.cache.scales.cpu().numpy()
    state = dl.state.buf.cpu().numpy()
    for s in seqs:
        a, b = int(wl.cu_seqlens[s]), int(wl.cu_seqlens[s + 1])
        h_v = O.bf16_decode(wl.hidden[a:b])
        rkv, rgate = O.project(h_v, w_v, D)
        err = _sum_error_bound(h_v, w_v)
        _bf16_close(gkv[a:b], rkv, err[:, :D], f"seq {s}: projected kv")
        _bf16_close(ggate[a:b], rgate, err[:, D:], f"seq {s}: projected gate")
        st = int(wl.start_pos[s])
        if b == a:  # no new token: nothing written
            continue
        O.compress_tokens(ol.main_state, ol.main_cache, s, st, O.bf16_decode(rkv), O.bf16_decode(rgate), ol.gamma,
                          1e-6, 64, 1e4)
        for blk in range(st // which, (st + b - a) // which):
            pg, sl = ol.main_cache.locate(s, blk)
            _rows_close_e2e(pages[pg, sl], scales[pg, sl], ol.main_cache.pages[pg, sl], ol.main_cache.scales[pg, sl],
                            spec.cache_dtype, f"seq {s} block {blk}")
        # the ring: each slot holds the kv and gate of the last token written to it (projected
        # values, or the initial state), within the projection's rule
        g = state[s].astype(np.float64)
        r = ol.main_state.buf[s].astype(np.float64)
        e = float(err.max()) if err.size else 0.0
        step = np.exp2(np.floor(np.log2(np.maximum(np.abs(r) + e, 2.0 ** -126))) - 7)
        assert np.all(np.abs(g - r) <= step + e), f"seq {s}: compressor state"
    return gkv, ggate


@pytest.mark.parametrize("m,D,cache_dtype", [(4, 128, "fp8"), (4, 128, "fp4"), (4, 512, "bf16"), (128, 512, "fp8")])
def test_compress_project_matches_oracle(m, D, cache_dtype):
    """Three sequences of 37, 300 and 129 tokens (several 128-token tiles, ragged tails, a
    sequence starting mid-block), hidden_dim 320 (five 64-wide slices)."""
    wl = W.projection_prefill(seed=31, lens=[37, 300, 129], start_pos=[0, 37, 5], hidden_dim=320, D=D,
                              cache_dtype=cache_dtype)
    _run(wl, m)


def test_compress_project_one_token_and_empty_sequence():
    """A single token (one partial 128-row tile) and a sequence with no new token."""
    wl = W.projection_prefill(seed=33, lens=[1, 0, 3], start_pos=[7, 4, 0], hidden_dim=64, D=128,
                              cache_dtype="bf16")
    _run(wl, 4)


@pytest.mark.slow
def test_compress_project_full_size():
    """The compressor-prefill workload with its projection: 8 sequences of 4096 tokens, hidden
    4096, D = 512 (two compressors' worth of weights, the C4 one run here); the oracle checks
    two of the sequences (first and last)."""
    wl = W.projection_prefill()
    _run(wl, 4, seqs=[0, 7])
