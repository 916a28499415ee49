"""Pins for the oracle: checks against things other than the oracle itself.

Each test ties one part of the oracle to a fixed point: the number-format
definitions (cross-checked with torch's casts), closed forms, hand-computed
values, invariants of the method, a library attention routine, brute force on
tiny inputs, and the KV-state sizing figures printed on the vLLM page.
"""

import itertools
import json
import math
import os

import mpmath
import numpy as np
import pytest
import torch

import oracle.dsv4_oracle as O

RNG = np.random.default_rng(1234)


# ----------------------------------------------------------------- codecs
def test_e4m3_decode_all_codes_match_library():
    codes = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    ours = O.e4m3_decode(codes)
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], lib[~nan])
    assert set(np.flatnonzero(nan)) == {0x7F, 0xFF}
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


def _fp32_cases(n):
    vals = O.E4M3_VALUES[:0x7F]
    mids = (vals[1:] + vals[:-1]) / 2  # exact ties
    x = np.concatenate([
        RNG.standard_normal(n) * 40.0,
        RNG.standard_normal(n) * 0.01,             # subnormal range
        RNG.uniform(-448, 448, n),
        mids, -mids, vals, -vals,
        np.nextafter(mids.astype(np.float32), np.float32(np.inf)),
        np.nextafter(mids.astype(np.float32), np.float32(-np.inf)),
    ]).astype(np.float32)
    return x


def test_e4m3_encode_matches_library_in_range():
    x = _fp32_cases(300_000)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode(x), lib)


def test_e4m3_encode_saturates_and_keeps_zero_sign():
    x = np.array([448.0, 449.0, 464.0, 1e30, -500.0, -1e-30, 1e-30, 0.0, -0.0], np.float32)
    got = O.e4m3_encode(x)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x80, 0x00, 0x00, 0x80]


def test_bf16_encode_matches_library():
    x = np.concatenate([RNG.standard_normal(200_000) * 10 ** RNG.uniform(-8, 8, 200_000),
                        (np.arange(1, 5000) * 2.0 ** -8 + 1.0 + 2.0 ** -9)]).astype(np.float32)
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.bf16_encode(x), lib)
    assert np.array_equal(O.bf16_decode(lib), torch.from_numpy(lib.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_fp8_store_scale_and_roundtrip():
    x = RNG.standard_normal(512) * 3.0
    codes, scale, dec = O.store(x, "fp8")
    amax = np.float32(np.max(np.abs(np.float32(x))))
    assert scale == np.float32(amax / np.float32(448.0))
    assert O.E4M3_VALUES[codes[np.argmax(np.abs(x))] & 0x7F] == 448.0
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range
    big = np.abs(x) > 2.0 ** -6 * float(scale)
    assert np.all(np.abs(dec[big] - x[big]) <= 2.0 ** -4 * np.abs(x[big]) + 1e-12)
    codes0, scale0, dec0 = O.store(np.zeros(8), "fp8")
    assert scale0 == 1.0 and np.all(codes0 == 0) and np.all(dec0 == 0)


# ----------------------------------------------------------------- pool / norm / rope
def test_gated_pool_closed_forms():
    kv = RNG.standard_normal((4, 6))
    # equal logits -> arithmetic mean
    assert np.allclose(O.gated_pool(kv, np.zeros((4, 6))), kv.mean(axis=0), atol=1e-15)
    # one token 60 above the rest -> that token, to within e^-60
    g = RNG.standard_normal((4, 6))
    g[2] += 60.0 + (g.max(axis=0) - g[2])
    assert np.max(np.abs(O.gated_pool(kv, g) - kv[2])) <= 4 * math.exp(-60) * np.max(np.abs(kv))
    # m = 1 -> identity
    assert np.allclose(O.gated_pool(kv[:1], g[:1]), kv[0], atol=0)
    # two tokens: hand-computed softmax weight
    kv2 = np.array([[1.0], [3.0]])
    g2 = np.array([[0.0], [math.log(3.0)]])  # weights 1/4, 3/4
    assert abs(O.gated_pool(kv2, g2)[0] - (0.25 * 1 + 0.75 * 3)) < 1e-15
    # scalar gate (G = 1) is the broadcast of a per-channel gate
    gs = RNG.standard_normal((4, 1))
    assert np.allclose(O.gated_pool(kv, gs), O.gated_pool(kv, np.repeat(gs, 6, axis=1)), atol=1e-15)
    # channels are independent: permuting channels permutes the output
    perm = RNG.permutation(6)
    assert np.allclose(O.gated_pool(kv[:, perm], g[:, perm]), O.gated_pool(kv, g)[perm])


def test_rms_norm_closed_forms():
    x = np.array([3.0, 4.0])
    assert np.allclose(O.rms_norm(x, np.ones(2), 0.0), x / math.sqrt(12.5), atol=1e-15)
    y = RNG.standard_normal(512)
    out = O.rms_norm(y, np.full(512, 2.5), 1e-6)
    assert abs(np.sqrt(np.mean(out ** 2)) - 2.5 * math.sqrt(np.mean(y ** 2) / (np.mean(y ** 2) + 1e-6))) < 1e-12
    assert np.allclose(O.rms_norm(7.0 * y, np.ones(512), 0.0), O.rms_norm(y, np.ones(512), 0.0), atol=1e-13)
    g = RNG.standard_normal(512)
    assert np.allclose(O.rms_norm(y, g, 0.0), O.rms_norm(y, np.ones(512), 0.0) * g, atol=1e-14)


def test_rope_hand_example():
    # D = 6, r = 4: dims 0,1 untouched; pairs (2,3) by pos*1, (4,5) by pos*10000^(-1/2)
    x = np.array([5.0, -7.0, 1.0, 0.0, 0.0, 1.0])
    y = O.apply_rope(x, 1, 4, 10000.0)
    want = np.array([5.0, -7.0, math.cos(1.0), math.sin(1.0), -math.sin(0.01), math.cos(0.01)])
    assert np.allclose(y, want, atol=1e-15)
    assert np.allclose(O.rope_inv_freq(4, 10000.0), [1.0, 0.01], atol=1e-18)


def test_rope_rotation_properties():
    x = RNG.standard_normal((3, 128))
    y = RNG.standard_normal((3, 128))
    for p in (0, 1, 4095, 131071, 1 << 20):
        r = O.apply_rope(x, p, 64, 10000.0)
        assert np.allclose(np.linalg.norm(r, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
        assert np.allclose(O.apply_rope(r, p, 64, 10000.0, inverse=True), x, atol=1e-12)
        assert np.array_equal(r[:, :64], x[:, :64])
    # <R_a x, R_b y> depends only on a - b
    a = np.einsum("ij,ij->i", O.apply_rope(x, 1000, 64, 1e4), O.apply_rope(y, 900, 64, 1e4))
    b = np.einsum("ij,ij->i", O.apply_rope(x, 100, 64, 1e4), O.apply_rope(y, 0, 64, 1e4))
    assert np.allclose(a, b, atol=1e-11)


def test_rope_angles_at_one_million_match_high_precision():
    mpmath.mp.dps = 40
    p, r = (1 << 20) + 7, 64
    x = np.zeros(r)
    x[0::2] = 1.0  # every pair = (1, 0) -> (cos a, sin a)
    y = O.apply_rope(x, p, r, 10000.0)
    for i in range(r // 2):
        a = mpmath.mpf(p) * mpmath.power(10000, mpmath.mpf(-2 * i) / r)
        assert abs(y[2 * i] - float(mpmath.cos(a))) < 1e-9
        assert abs(y[2 * i + 1] - float(mpmath.sin(a))) < 1e-9


# ----------------------------------------------------------------- compressor
def _cache(m, D, dtype, B=1, blocks=8, seed=0):
    rng = np.random.default_rng(seed)
    pp = O.PAGE_POSITIONS // m
    num_pages = B * blocks + 2
    bt = rng.permutation(num_pages)[: B * blocks].reshape(B, blocks).astype(np.int32)
    pages = np.zeros((num_pages, pp, D), dtype=O.CODE_DTYPE[dtype])
    return O.PagedCache(dtype, m, D, pages, np.ones((num_pages, pp), np.float32), bt)


def test_compressor_streaming_is_chunking_invariant():
    m, D, T = 4, 16, 61
    kv = RNG.standard_normal((T, D)).astype(np.float32)
    g = RNG.standard_normal((T, D)).astype(np.float32)
    gamma = 1 + 0.1 * RNG.standard_normal(D)
    outs = []
    for cuts in ([0, T], [0, 37, T], list(range(T + 1))):
        st = O.CompressorState(m, D, D, np.zeros((1, m, 2 * D), np.float32))
        c = _cache(m, D, "f32")
        for a, b in zip(cuts[:-1], cuts[1:]):
            O.compress_tokens(st, c, 0, a, kv[a:b], g[a:b], gamma, 1e-6, 8, 1e4)
        outs.append((c.read(0, np.arange(T // m)), st.buf.copy()))
    for e, s in outs[1:]:
        assert np.array_equal(e, outs[0][0]) and np.array_equal(s, outs[0][1])
    # the ring keeps the last T % m tokens in their slots
    tail = np.arange(T - T % m, T)
    assert np.array_equal(outs[0][1][0, tail % m, :D], kv[tail])
    # entry b is exactly the formula on tokens 4b..4b+3
    b = 9
    want = O.apply_rope(O.rms_norm(O.gated_pool(kv[4 * b:4 * b + 4], g[4 * b:4 * b + 4]), gamma, 1e-6),
                        4 * b, 8, 1e4)
    assert np.allclose(outs[0][0][b], O.f32(want), atol=0)


def test_compress_block_with_m1_is_the_window_key():
    kv = RNG.standard_normal(32)
    gamma = RNG.standard_normal(32)
    for t in (0, 5, 1000):
        a = O.compress_block(kv[None], RNG.standard_normal((1, 32)), t, 1, gamma, 1e-6, 16, 1e4)
        assert np.allclose(a, O.window_key(kv, t, gamma, 1e-6, 16, 1e4), atol=1e-14)


# ----------------------------------------------------------------- indexer / top-k
def test_indexer_scores_brute_force():
    q = RNG.standard_normal((3, 5))
    w = RNG.standard_normal(3)
    k = RNG.standard_normal((7, 5))
    want = []
    for j in range(7):
        s = 0.0
        for h in range(3):
            dot = sum(q[h, c] * k[j, c] for c in range(5))
            s += w[h] * (dot if dot > 0 else 0.0)
        want.append(s)
    assert np.allclose(O.indexer_scores(q, w, k), want, atol=1e-14)
    # every q.k < 0 -> every score is 0 (a full tie)
    kneg = -np.abs(k)
    assert np.all(O.indexer_scores(np.abs(q), w, kneg) == 0.0)


def _check_topk_property(s, k, idx):
    n = len(s)
    sel = [int(j) for j in idx if j >= 0]
    assert len(sel) == min(k, n) and len(set(sel)) == len(sel)
    assert all(j == -1 for j in idx[len(sel):])
    rest = set(range(n)) - set(sel)
    for a in sel:
        for b in rest:
            assert s[a] > s[b] or (s[a] == s[b] and a < b)


def test_topk_selection_property_and_ties():
    for n, k in ((50, 7), (5, 8), (64, 64), (200, 17)):
        s = RNG.integers(-3, 4, n).astype(np.float64)  # many exact ties
        _check_topk_property(s, k, O.topk_select(s, k))
        s = RNG.standard_normal(n)
        _check_topk_property(s, k, O.topk_select(s, k))
    # brute force over all subsets on a tiny case
    s = np.array([0.5, 2.0, 2.0, -1.0, 0.5, 3.0])
    best = max(itertools.combinations(range(6), 3), key=lambda c: sorted(((s[j], -j) for j in c), reverse=True))
    assert set(O.topk_select(s, 3)) == set(best) == {5, 1, 2}
    assert list(O.topk_select(np.zeros(5), 3)) == [0, 1, 2]


# ----------------------------------------------------------------- attention
def test_shared_kv_attention_matches_library_sdpa():
    H, D, N, r = 8, 64, 37, 32
    q = RNG.standard_normal((H, D))
    keys = RNG.standard_normal((N, D))
    p = 12345
    tau = 1 / math.sqrt(D)
    got = O.shared_kv_attention(q, p, keys, tau, r, 1e4)
    qr = torch.from_numpy(O.apply_rope(q, p, r, 1e4))[None, :, None, :]  # [1, H, 1, D]
    K = torch.from_numpy(keys)[None, None].expand(1, H, N, D)
    o = torch.nn.functional.scaled_dot_product_attention(qr, K, K, scale=tau)[0, :, 0].numpy()
    assert np.allclose(got, O.apply_rope(o, p, r, 1e4, inverse=True), atol=1e-12)


def _tiny_layer(kind, m, W, k, D=32, H=4, B=1, ctx_blocks=8, d_I=8, H_I=2):
    cfg = O.LayerConfig(kind=kind, m=m, H=H, D=D, W=W, k=k, H_I=H_I, d_I=d_I, rope_dims=16,
                        idx_rope_dims=4, eps=1e-6)
    st = O.LayerState(cfg=cfg, gamma=1 + 0.1 * RNG.standard_normal(D),
                      main_state=O.CompressorState(m, D, D, np.zeros((B, m, 2 * D), np.float32)),
                      main_cache=_cache(m, D, "f32", B, ctx_blocks),
                      window=O.WindowRing("f32", W, D, np.zeros((B, W, D), np.float32), np.ones((B, W), np.float32)))
    if kind == "c4":
        st.gamma_idx = np.ones(d_I)
        st.idx_state = O.CompressorState(m, d_I, d_I, np.zeros((B, m, 2 * d_I), np.float32))
        st.idx_cache = _cache(m, d_I, "f32", B, ctx_blocks, seed=1)
    return st


def _run_tokens(layer, T):
    """Decode T tokens one at a time; return inputs of the last step."""
    c = layer.cfg
    for t in range(T):
        step = O.StepInputs(pos=np.array([t]), kv=RNG.standard_normal((1, c.D)),
                            gate=RNG.standard_normal((1, c.D)), q=RNG.standard_normal((1, c.H, c.D)),
                            q_idx=RNG.standard_normal((1, c.H_I, c.d_I)), w=RNG.standard_normal((1, c.H_I)),
                            idx_kv=RNG.standard_normal((1, c.d_I)), idx_gate=RNG.standard_normal((1, c.d_I)))
        O.decode_update(layer, step)
    return step


def test_inverse_rope_end_to_end_single_key():
    # only the current token is visible: n_c = floor(6/128) = 0, W = 1
    layer = _tiny_layer("c128", 128, 1, 0)
    step = _run_tokens(layer, 6)
    o, sel, _ = O.decode_attend(layer, step)[0]
    want = O.rms_norm(O.f32(O.f32(step.kv[0])), layer.gamma, 1e-6)  # window stores float32
    assert sel.shape[0] == 0
    assert np.allclose(o, np.broadcast_to(want, o.shape), atol=2e-6)


def test_window_covering_context_is_dense_causal_attention():
    # C128 with p+1 < m: no compressed entry, window >= p+1 -> causal attention over all raw keys
    layer = _tiny_layer("c128", 128, 64, 0)
    T = 40
    kvs = []
    c = layer.cfg
    for t in range(T):
        step = O.StepInputs(pos=np.array([t]), kv=RNG.standard_normal((1, c.D)),
                            gate=RNG.standard_normal((1, c.D)), q=RNG.standard_normal((1, c.H, c.D)))
        O.decode_update(layer, step)
        kvs.append(step.kv[0])
    keys = np.stack([O.f32(O.window_key(kv, t, layer.gamma, 1e-6, 16, 1e4)) for t, kv in enumerate(kvs)])
    o, _, _ = O.decode_attend(layer, step)[0]
    qr = torch.from_numpy(O.apply_rope(step.q[0], T - 1, 16, 1e4))[None, :, None, :]
    K = torch.from_numpy(keys.astype(np.float64))[None, None].expand(1, c.H, T, c.D)
    ref = torch.nn.functional.scaled_dot_product_attention(qr, K, K, scale=c.tau)[0, :, 0].numpy()
    assert np.allclose(o, O.apply_rope(ref, T - 1, 16, 1e4, inverse=True), atol=1e-12)


def test_topk_covering_all_entries_is_dense_over_window_and_entries():
    # C4 with k >= n_c and W >= p+1: attention over window U all compressed entries
    layer = _tiny_layer("c4", 4, 64, 64)
    step = _run_tokens(layer, 43)
    p = 42
    n_c = O.visible_entries(p, 4)
    assert n_c == 10
    o, sel, _ = O.decode_attend(layer, step)[0]
    assert sorted(sel) == list(range(n_c))
    keys = np.concatenate([layer.window.read(0, np.arange(0, p + 1)), layer.main_cache.read(0, np.arange(n_c))])
    assert np.allclose(o, O.shared_kv_attention(step.q[0], p, keys, layer.cfg.tau, 16, 1e4), atol=1e-13)
    # m = 1 compression is the identity on raw keys: entries equal window keys
    l1 = _tiny_layer("c4", 1, 64, 64)
    _run_tokens(l1, 20)
    assert np.allclose(l1.main_cache.read(0, np.arange(20)), l1.window.read(0, np.arange(20)), atol=0)


def test_visible_counts_of_the_workloads(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "layer_shapes.json")))
    assert g["page_positions"] == O.PAGE_POSITIONS
    # the decode token at position L sees floor((L+1)/m) complete blocks
    assert O.visible_entries(4096, g["c4_ratio"]) == 1024
    assert O.visible_entries(65536, g["c128_ratio"]) == 512
    assert O.visible_entries(131072, g["c4_ratio"]) == 32768
    assert O.visible_entries(1 << 20, g["c4_ratio"]) == 262144
    assert O.visible_entries(1 << 20, g["c128_ratio"]) == 8192
    assert O.visible_entries((1 << 20) + 3, 4) == 262145   # first new C4 entry at step 3
    assert list(O.window_positions(5, g["swa_window"])) == list(range(6))
    assert len(O.window_positions(10_000, g["swa_window"])) == 128


# ----------------------------------------------------------------- sizing
def test_kv_state_sizing_reproduces_the_page(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "kv_state_sizing.json")))
    L = g["context_tokens"]
    gib = float(1 << 30)
    v32 = O.kv_state_bytes(L, [(1, 576 + 128, 0, 0)] * 61, g["bytes_per_value"]) / gib
    v4 = O.kv_state_bytes(L, [(4, 512 + 128, 0, 0)] * 30 + [(128, 512, 0, 0)] * 31, g["bytes_per_value"]) / gib
    assert round(v32, 1) == g["v32_gib"]
    assert round(v4, 2) == g["v4_gib"]
    assert round(v32 / v4, 1) == g["ratio"]


# ----------------------------------------------------------------- query norm, fp8 output
def test_query_norm_closed_form_and_scale_invariance():
    """R21: with gamma = 1 every normed head has RMS 1 (up to eps); the attention then does not
    depend on a positive per-head scale of the query."""
    H, D, N = 4, 64, 23
    q = RNG.standard_normal((H, D)) * np.array([[0.5], [3.0], [10.0], [0.1]])
    qn = O.query_norm(q, np.ones(D), 1e-6)
    ms = np.mean(q * q, axis=1)
    assert np.allclose(np.sqrt(np.mean(qn * qn, axis=1)), np.sqrt(ms / (ms + 1e-6)), rtol=1e-12)
    keys = RNG.standard_normal((N, D))
    scale = np.array([[7.0], [0.25], [1.0], [40.0]])
    a = O.shared_kv_attention(O.query_norm(q, np.ones(D), 0.0), 99, keys, 0.125, 16, 1e4)
    b = O.shared_kv_attention(O.query_norm(q * scale, np.ones(D), 0.0), 99, keys, 0.125, 16, 1e4)
    assert np.allclose(a, b, atol=1e-12)


def test_fp8_output_blocks_hand_example():
    """R22: every 128-channel block gets its own scale amax/448; a block's largest value maps
    to code 448 (0x7E), and the blocks do not see each other."""
    o = np.zeros((2, 256))
    o[0, :128] = np.linspace(-1.0, 1.0, 128)       # amax 1
    o[0, 128:] = 1e-3 * np.linspace(0.0, 2.0, 128)  # amax 2e-3
    o[1, :] = 448.0 * 4                             # amax 1792, constant
    codes, scales, dec = O.store_output(o, "fp8")
    assert scales.shape == (2, 2)
    assert scales[0, 0] == np.float32(np.float32(1.0) / np.float32(448.0))
    assert scales[0, 1] == np.float32(np.float32(2e-3) / np.float32(448.0))
    assert scales[1, 0] == scales[1, 1] == np.float32(4.0)
    assert codes[0, 127] == 0x7E and codes[0, 0] == 0xFE and codes[0, 255] == 0x7E
    assert np.all(codes[1] == 0x7E) and np.all(dec[1] == 1792.0)
    # the small block keeps its relative precision (its own scale), e4m3: 2^-4 relative
    big = np.abs(o[0, 128:]) > 2.0 ** -6 * float(scales[0, 1])
    assert np.all(np.abs(dec[0, 128:][big] - o[0, 128:][big]) <= 2.0 ** -4 * np.abs(o[0, 128:][big]))
    # against the library cast of the scaled block
    inv = np.float32(np.float32(448.0) / np.float32(1.0))
    lib = torch.from_numpy(np.float32(o[0, :128]).astype(np.float32) * inv).to(torch.float8_e4m3fn)
    assert np.array_equal(codes[0, :128], lib.view(torch.uint8).numpy())


# ----------------------------------------------------------------- fp4 indexer cache (R23)
def test_e2m1_codes_from_the_format_definition():
    """All 16 e2m1 codes: the OCP E2M1 table (sign, 2 exponent bits with bias 1, 1 mantissa
    bit), written out by hand."""
    table = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert list(O.E2M1_VALUES[:8]) == table
    assert list(O.E2M1_VALUES[8:]) == [-v for v in table]
    assert np.signbit(O.E2M1_VALUES[8])


def test_e2m1_encode_is_nearest_with_ties_to_even():
    """Against brute force: the nearest of the 8 magnitudes, an exact tie going to the code
    with an even mantissa bit; saturation at 6; the sign kept, also for values rounding to 0."""
    x = np.concatenate([RNG.uniform(-8, 8, 20000), np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25,
                                                              -5.0, 7.0, -100.0, 1e-9, -1e-9, 0.0])]).astype(np.float32)
    got = O.e2m1_encode(x)
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    for v, c in zip(x.astype(np.float64), got):
        a = min(abs(v), 6.0)
        d = np.abs(mags - a)
        best = np.flatnonzero(d == d.min())
        want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        assert (c & 7) == want and bool(c & 8) == bool(np.signbit(v)), (v, c)
    # the hand-picked ties
    assert list(O.e2m1_encode(np.float32([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]))) == [0, 2, 2, 4, 4, 6, 6]


def test_fp4_rows_pack_and_scale():
    x = RNG.standard_normal(128) * 2.0
    packed, scale, dec = O.store(x, "fp4")
    assert packed.shape == (64,) and packed.dtype == np.uint8
    amax = np.float32(np.max(np.abs(np.float32(x))))
    assert scale == np.float32(amax / np.float32(6.0))
    codes = O.fp4_unpack(packed)
    assert np.array_equal(O.fp4_pack(codes), packed)
    assert codes[np.argmax(np.abs(x))] & 7 == 7  # the largest value maps to 6
    assert np.array_equal(dec, O.decode_rows(packed[None], np.array([scale]), "fp4")[0])
    # even elements in the low nibble
    p2 = O.fp4_pack(np.array([3, 12], np.uint8))
    assert p2[0] == 0xC3
    # e2m1 keeps 1 mantissa bit: relative error <= 1/4 above the subnormal range
    big = np.abs(x) >= float(scale)
    assert np.all(np.abs(dec[big] - x[big]) <= 0.25 * np.abs(x[big]) + 1e-12)


# ----------------------------------------------------------------- projection (R24)
def _bf16_neighbours(v: float):
    """The two bf16 values around v (v itself twice when v is one), from the bit patterns."""
    f = np.float32(v)
    u = int(np.array([f]).view(np.uint32)[0])
    lo_bits = u & 0xFFFF0000
    lo = float(np.array([lo_bits], np.uint32).view(np.float32)[0])
    hi = float(np.array([lo_bits + 0x10000], np.uint32).view(np.float32)[0])
    return (lo, hi) if abs(lo) <= abs(v) else (hi, lo)


def test_bf16_round_exact_is_nearest_ties_to_even():
    # hand ties: halfway between 1 and 1 + 2^-7 goes to 1 (even), halfway above goes up
    got = O.bf16_round_exact(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 3.0, 0.0]))
    assert list(got) == [1.0, 1 + 2.0 ** -6, -1.0, 3.0, 0.0]
    # random values against the two neighbouring bf16 values, chosen by distance (float64 values
    # that float32 would round first are included: the rounding is from the exact value)
    xs = np.concatenate([RNG.standard_normal(3000) * 10.0 ** RNG.integers(-3, 4, 3000),
                         1 + (2 * RNG.integers(0, 64, 200) + 1) * 2.0 ** -8 + 2.0 ** -40])
    for v, r in zip(xs, O.bf16_round_exact(xs)):
        a, b = sorted(_bf16_neighbours(v), key=abs)
        da, db = abs(v - a), abs(v - b)
        assert r == (a if da < db else b if db < da else r), (v, r, a, b)
        assert r in (a, b)


def test_projection_brute_force_and_closed_forms():
    # brute force: every output element as an explicit sum over the hidden dim
    T, Hd, D = 3, 5, 2
    h = RNG.standard_normal((T, Hd))
    w = RNG.standard_normal((2 * D, Hd))
    kv, gate = O.project(h, w, D)
    for t in range(T):
        for c in range(2 * D):
            acc = 0.0
            for i in range(Hd):
                acc += h[t, i] * w[c, i]
            want = O.bf16_round_exact(acc)
            got = O.bf16_decode(kv[t, c] if c < D else gate[t, c - D])
            assert got == want, (t, c)
    # identity weights: kv is the hidden state, gate twice it, each rounded to bf16
    h2 = RNG.standard_normal((4, 8))
    kv2, gate2 = O.project(h2, np.vstack([np.eye(8), 2 * np.eye(8)]), 8)
    assert np.array_equal(O.bf16_decode(kv2), O.bf16_round_exact(h2))
    assert np.array_equal(O.bf16_decode(gate2), O.bf16_round_exact(2 * h2))
    # scaling the hidden state by a power of two scales the output exactly
    kv3, _ = O.project(4.0 * h2, np.vstack([np.eye(8), np.eye(8)]), 8)
    assert np.array_equal(O.bf16_decode(kv3), 4.0 * O.bf16_decode(kv2))


def test_e2m1_encode_matches_library_cast():
    """The e2m1 encoder against ml_dtypes' float4_e2m1fn cast (round to nearest even,
    saturating at 6) on random values inside and beyond the range, and signed zeros."""
    ml_dtypes = pytest.importorskip("ml_dtypes")
    x = np.concatenate([RNG.uniform(-7.5, 7.5, 50000), RNG.standard_normal(20000) * 3,
                        np.array([0.0, -0.0, 6.0, -6.0, 6.5, -9.0, 0.2, -0.2])]).astype(np.float32)
    ours = O.e2m1_decode(O.e2m1_encode(x))
    lib = x.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(ours, lib)
    assert np.array_equal(np.signbit(ours[ours == 0]), np.signbit(lib[lib == 0]))
