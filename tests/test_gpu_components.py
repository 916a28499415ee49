"""GPU parity of each entry point of the C ABI against the oracle, on the same bytes.

Sizes span several tiles with ragged tails; edge cases: unaligned prefill starts,
truncated windows, n_c = 0, n_c <= k, full score ties, -1 padding and an
out-of-range index in the selection.
"""

import numpy as np
import pytest
import torch

import compressed_sparse_kv_dsv4_b200 as dsv4
import oracle.dsv4_oracle as O
import synthetic as W
from oracle import adapters as OA
from tests.parity import (check_output, check_output_fp8, check_topk, codes_close, decode_out, input_class,
                          require_gpu)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


# ---------------------------------------------------------------------------- compressor
@pytest.mark.parametrize("m,cache_dtype,D", [(4, "bf16", 512), (128, "fp8", 512), (4, "fp8", 128), (4, "f32", 32),
                                               (4, "fp4", 128)])
def test_compress_prefill_matches_oracle(m, cache_dtype, D):
    rng = W.rng_for(11)
    lens = np.array([37, 300, 129], dtype=np.int32)
    start = np.array([0, 37, 5], dtype=np.int32)
    if m == 128:
        lens = np.array([300, 129, 411], dtype=np.int32)
        start = np.array([0, 200, 5], dtype=np.int32)
    B = len(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    T = int(cu[-1])
    kv_dt = "f32" if cache_dtype == "f32" else "bf16"
    kv = W.encode_values(W.normal_f32(rng, (T, D)), kv_dt)
    gate = W.encode_values(W.normal_f32(rng, (T, D)), kv_dt)
    spec = W.LayerSpec(kind="c128", m=m, H=8, D=D, cache_dtype=cache_dtype, kv_dtype=kv_dt, swa_dtype="bf16")
    la = W.make_layer(spec, B, int((start + lens).max()) // m + 1, seed=5)
    la.gamma = (1 + 0.2 * W.normal_f32(rng, (D,))).astype(np.float32)
    dl = dsv4.DeviceLayer.from_arrays(la)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dsv4.compress(dsv4.to_device_codes(kv, kv_dt, "cuda"), dsv4.to_device_codes(gate, kv_dt, "cuda"),
                  torch.from_numpy(cu).cuda(), torch.from_numpy(start).cuda(), dl.state, dl.cache, dl.gamma,
                  kv_dtype=kv_dt, eps=1e-6, rope_dims=min(64, D // 2), rope_base=1e4, d_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ol = OA.layer_state(la)
    dec = lambda a: OA.decode_input(a, kv_dt)  # noqa: E731
    O.compress(dec(kv), dec(gate), cu, start, ol.main_state, ol.main_cache, ol.gamma, 1e-6, min(64, D // 2), 1e4)
    # the state ring holds exact copies of the inputs
    assert np.array_equal(dl.state.buf.cpu().numpy(), ol.main_state.buf)
    pages = dsv4.to_numpy_codes(dl.cache.pages, cache_dtype)
    scales = dl.cache.scales.cpu().numpy()
    for s in range(B):
        for b in range(start[s] // m, (start[s] + lens[s]) // m):
            pg, sl = ol.main_cache.locate(s, b)
            codes_close(pages[pg, sl], ol.main_cache.pages[pg, sl], scales[pg, sl], ol.main_cache.scales[pg, sl],
                         cache_dtype, f"seq {s} block {b}")
    # rows that no block wrote keep their bytes
    untouched = np.ones(pages.shape[:2], bool)
    for s in range(B):
        for b in range(start[s] // m, (start[s] + lens[s]) // m):
            untouched[ol.main_cache.locate(s, b)] = False
    assert np.array_equal(pages[untouched], la.pages[untouched])


def test_compress_prefill_equals_token_by_token():
    rng = W.rng_for(12)
    D, m, T = 128, 4, 77
    kv = W.bf16_bits(W.normal_f32(rng, (T, D)))
    gate = W.bf16_bits(W.normal_f32(rng, (T, D)))
    spec = W.LayerSpec(kind="c128", m=m, H=8, D=D, cache_dtype="fp8", kv_dtype="bf16")
    la = W.make_layer(spec, 1, T // m + 1, seed=6)
    outs = []
    for chunks in ([T], [1] * T, [37, 40]):
        dl = dsv4.DeviceLayer.from_arrays(la)
        kvd = dsv4.to_device_codes(kv, "bf16", "cuda")
        gd = dsv4.to_device_codes(gate, "bf16", "cuda")
        p0 = 0
        for c in chunks:
            dsv4.compress(kvd[p0:p0 + c], gd[p0:p0 + c], torch.tensor([0, c], dtype=torch.int32, device="cuda"),
                          torch.tensor([p0], dtype=torch.int32, device="cuda"), dl.state, dl.cache, dl.gamma,
                          kv_dtype="bf16", rope_dims=64)
            p0 += c
        torch.cuda.synchronize()
        outs.append((dl.cache.pages.cpu().numpy(), dl.cache.scales.cpu().numpy(), dl.state.buf.cpu().numpy()))
    for o in outs[1:]:
        for a, b in zip(o, outs[0]):
            assert np.array_equal(a, b)


@pytest.mark.slow
@pytest.mark.parametrize("cache_dtype", ["bf16", "fp8"])
def test_compressor_prefill_full_size(cache_dtype):
    """The compressor prefill workload at full size: 8 sequences of 4096 bf16 tokens (D = 512)
    into a C4 and a C128 compressor. Checked against the oracle: every C128 entry (256), a
    seeded sample of 320 C4 entries (every sequence's first and last among them), and both
    state rings, which end holding each sequence's last block of inputs."""
    wl = W.compressor_prefill(cache_dtype=cache_dtype)
    B = wl.start_pos.shape[0]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cu = torch.from_numpy(wl.cu_seqlens).cuda()
    sp = torch.from_numpy(wl.start_pos).cuda()
    rng = np.random.default_rng(71)
    for la, kv, gate in ((wl.layer4, wl.kv4, wl.gate4), (wl.layer128, wl.kv128, wl.gate128)):
        spec = la.spec
        m = spec.m
        dl = dsv4.DeviceLayer.from_arrays(la)
        dsv4.compress(dsv4.to_device_codes(kv, "bf16", "cuda"), dsv4.to_device_codes(gate, "bf16", "cuda"), cu, sp,
                      dl.state, dl.cache, dl.gamma, kv_dtype="bf16", eps=spec.eps, rope_dims=spec.rope_dims,
                      rope_base=spec.rope_base, d_status=status)
        torch.cuda.synchronize()
        assert status.item() == 0
        ol = OA.layer_state(la)
        pages = dsv4.to_numpy_codes(dl.cache.pages, cache_dtype)
        scales = dl.cache.scales.cpu().numpy()
        n_blocks = [(int(wl.cu_seqlens[s + 1] - wl.cu_seqlens[s]) + int(wl.start_pos[s])) // m for s in range(B)]
        if m == 128:
            pairs = [(s, b) for s in range(B) for b in range(n_blocks[s])]
        else:
            pairs = {(s, b) for s in range(B) for b in (0, n_blocks[s] - 1)}
            while len(pairs) < 320:
                s = int(rng.integers(B))
                pairs.add((s, int(rng.integers(n_blocks[s]))))
            pairs = sorted(pairs)
        for s, b in pairs:
            t0 = int(wl.cu_seqlens[s]) + b * m - int(wl.start_pos[s])
            e = O.compress_block(OA.decode_input(kv[t0:t0 + m], "bf16"), OA.decode_input(gate[t0:t0 + m], "bf16"),
                                 b, m, ol.gamma, spec.eps, spec.rope_dims, spec.rope_base)
            codes, scale, _ = O.store(e, cache_dtype)
            pg, sl = ol.main_cache.locate(s, b)
            codes_close(pages[pg, sl], codes, scales[pg, sl], scale, cache_dtype, f"m={m} seq {s} entry {b}",
                        max_frac=0.05)
        ring = dl.state.buf.cpu().numpy()
        for s in range(B):
            t_end = int(wl.cu_seqlens[s + 1])
            for i in range(m):  # the ring slot of each of the last m positions holds its inputs
                t = t_end - m + i
                p = t - int(wl.cu_seqlens[s]) + int(wl.start_pos[s])
                want = np.concatenate([OA.decode_input(kv[t], "bf16"), OA.decode_input(gate[t], "bf16")])
                assert np.array_equal(ring[s, p % m], want.astype(np.float32)), f"m={m} seq {s} ring slot {p % m}"


@pytest.mark.parametrize("dtype,D", [("fp8", 512), ("bf16", 512), ("f32", 128)])
def test_swa_insert_matches_oracle(dtype, D):
    rng = W.rng_for(13)
    lens = np.array([5, 200, 128], dtype=np.int32)
    start = np.array([0, 1000, 70], dtype=np.int32)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    kv_dt = "f32" if dtype == "f32" else "bf16"
    kv = W.encode_values(W.normal_f32(rng, (int(cu[-1]), D)), kv_dt)
    spec = W.LayerSpec(kind="c128", m=128, H=8, D=D, swa_dtype=dtype, cache_dtype="bf16", kv_dtype=kv_dt)
    la = W.make_layer(spec, 3, 4, seed=7)
    la.gamma = (1 + 0.2 * W.normal_f32(rng, (D,))).astype(np.float32)
    dl = dsv4.DeviceLayer.from_arrays(la)
    dsv4.swa_insert(dsv4.to_device_codes(kv, kv_dt, "cuda"), torch.from_numpy(cu).cuda(),
                    torch.from_numpy(start).cuda(), dl.ring, dl.gamma, kv_dtype=kv_dt, rope_dims=64)
    torch.cuda.synchronize()
    ol = OA.layer_state(la)
    kvf = OA.decode_input(kv, kv_dt)
    for s in range(3):
        for i in range(lens[s]):
            t = start[s] + i
            if t >= start[s] + lens[s] - 128:
                O.swa_insert(ol.window, s, t, kvf[cu[s] + i], ol.gamma, 1e-6, 64, 1e4)
    rows = dsv4.to_numpy_codes(dl.ring.rows, dtype)
    sc = dl.ring.scales.cpu().numpy()
    for s in range(3):
        for i in range(128):
            codes_close(rows[s, i], ol.window.rows[s, i], sc[s, i], ol.window.scales[s, i], dtype, f"seq {s} slot {i}")


# ---------------------------------------------------------------------------- indexer
def _indexer_case(n_list, k, H=64, seed=21, spec=W.C4_SPEC, all_negative=False):
    B = len(n_list)
    la = W.make_layer(spec, B, max(n_list) + 1, seed, outlier_frac=0.05)
    st = W.make_step(spec, B, 0, seed + 1)
    if all_negative:  # every q.k < 0: all scores are exactly zero
        st.q_idx = st.q_idx & 0x7F
        # the sign bit of every key element: bit 7 of an e4m3 code, bit 3 of each e2m1 nibble
        la.idx_pages = la.idx_pages | (0x88 if spec.idx_dtype == "fp4" else 0x80)
    dl = dsv4.DeviceLayer.from_arrays(la)
    q = dsv4.to_device_codes(st.q_idx, spec.q_idx_dtype, "cuda")
    w = dsv4.to_device_codes(st.w, spec.w_dtype, "cuda")
    n = torch.tensor(n_list, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx, scores = dsv4.indexer_topk(q, w, dl.idx_cache, n, k, q_dtype=spec.q_idx_dtype, w_dtype=spec.w_dtype,
                                    q_scale=torch.from_numpy(st.q_idx_scale).cuda(), d_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ol = OA.layer_state(la)
    qd = OA.decode_input(st.q_idx, spec.q_idx_dtype, st.q_idx_scale)
    wd = OA.decode_input(st.w, spec.w_dtype)
    return idx.cpu().numpy(), scores.cpu().numpy(), ol, qd, wd


@pytest.mark.parametrize("k", [512, 64, 1024])
def test_indexer_tensor_core_topk_matches_oracle(k):
    n_list = [130, 1000, 4097, 0, 600]
    idx, scores, ol, qd, wd = _indexer_case(n_list, k)
    for s, n in enumerate(n_list):
        if n == 0:
            assert np.all(idx[s] == -1)
            continue
        ref = O.indexer_scores(qd[s], wd[s], ol.idx_cache.read(s, np.arange(n)))
        check_topk(idx[s], ref, k, n, f"seq {s}")
        v = idx[s] >= 0
        got = scores[s][v]
        want = ref[idx[s][v]]
        assert np.all(np.abs(got - want) <= 1e-5 * np.abs(want).max()), f"seq {s}: scores"


def test_indexer_tensor_core_fp4_keys_topk_matches_oracle():
    """e2m1 keys (two per byte, one float32 scale per row) against fp8 queries, on the tensor
    cores: scores and the top-k set equal the oracle's on the same codes."""
    n_list = [130, 1000, 4097, 0, 600, 20000]
    idx, scores, ol, qd, wd = _indexer_case(n_list, 512, seed=27, spec=W.C4_FP4_SPEC)
    for s, n in enumerate(n_list):
        if n == 0:
            assert np.all(idx[s] == -1)
            continue
        ref = O.indexer_scores(qd[s], wd[s], ol.idx_cache.read(s, np.arange(n)))
        check_topk(idx[s], ref, 512, n, f"seq {s}")
        v = idx[s] >= 0
        assert np.all(np.abs(scores[s][v] - ref[idx[s][v]]) <= 1e-5 * np.abs(ref).max()), f"seq {s}: scores"


def test_indexer_tensor_core_long_sequences_topk_matches_oracle():
    """Sequences of 46K-70K entries: top-k clusters of more CTAs, slices of 24 keys per
    thread, an empty sequence beside them."""
    n_list = [50000, 46100, 0, 70001]
    idx, scores, ol, qd, wd = _indexer_case(n_list, 512, seed=23)
    for s, n in enumerate(n_list):
        if n == 0:
            assert np.all(idx[s] == -1)
            continue
        ref = O.indexer_scores(qd[s], wd[s], ol.idx_cache.read(s, np.arange(n)))
        check_topk(idx[s], ref, 512, n, f"seq {s}")


def test_indexer_many_short_sequences_topk_in_entry_order():
    """48 sequences of 0 to 5000 entries (several per CTA of the scoring kernel), many with
    fewer entries than k: the selection pads with -1 and writes the kept entries in ascending
    entry order."""
    n_list = [3, 700, 64, 5000, 1, 130, 0, 257] * 6
    idx, scores, ol, qd, wd = _indexer_case(n_list, 64, seed=25)
    for s, n in enumerate(n_list):
        ref = O.indexer_scores(qd[s], wd[s], ol.idx_cache.read(s, np.arange(n))) if n else np.zeros(0)
        check_topk(idx[s], ref, 64, n, f"seq {s}")
        v = idx[s] >= 0
        assert np.all(np.diff(idx[s][v]) > 0), f"seq {s}: output not in ascending entry order"


@pytest.mark.parametrize("idx_dtype", ["fp8", "fp4"])
def test_indexer_scores_alone_match_oracle(idx_dtype):
    """dsv4_indexer_scores: every visible entry's score (the tensor-core kernel alone), rows
    past n_entries untouched."""
    spec = W.C4_FP4_SPEC if idx_dtype == "fp4" else W.C4_SPEC
    n_list = [130, 4097, 0, 600]
    B = len(n_list)
    la = W.make_layer(spec, B, max(n_list) + 1, 24, outlier_frac=0.05)
    st = W.make_step(spec, B, 0, 25)
    dl = dsv4.DeviceLayer.from_arrays(la)
    out = dsv4.indexer_scores(dsv4.to_device_codes(st.q_idx, "fp8", "cuda"), dsv4.to_device_codes(st.w, "bf16", "cuda"),
                              dl.idx_cache, torch.tensor(n_list, dtype=torch.int32, device="cuda"), q_dtype="fp8",
                              w_dtype="bf16", q_scale=torch.from_numpy(st.q_idx_scale).cuda())
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    ol = OA.layer_state(la)
    qd = OA.decode_input(st.q_idx, spec.q_idx_dtype, st.q_idx_scale)
    wd = OA.decode_input(st.w, spec.w_dtype)
    for s_, n in enumerate(n_list):
        assert np.all(np.isnan(got[s_, n:])), f"seq {s_}: entries past n_entries were written"
        if n:
            ref = O.indexer_scores(qd[s_], wd[s_], ol.idx_cache.read(s_, np.arange(n)))
            assert np.all(np.abs(got[s_, :n] - ref) <= 1e-5 * np.abs(ref).max()), f"seq {s_}"


@pytest.mark.parametrize("idx_dtype", ["fp8", "fp4"])
def test_indexer_full_tie_takes_lowest_indices(idx_dtype):
    spec = W.C4_FP4_SPEC if idx_dtype == "fp4" else W.C4_SPEC
    idx, scores, ol, qd, wd = _indexer_case([3000, 700], 512, all_negative=True, spec=spec)
    for s in range(2):
        assert sorted(idx[s].tolist()) == list(range(512))
        assert np.all(scores[s] == 0.0)


def test_indexer_cuda_core_path_fp32_with_query_rope():
    spec = W.TINY_SPEC
    B, n = 2, 1024
    la = W.make_layer(spec, B, n + 1, 31)
    st = W.make_step(spec, B, [4096, 777], 32)
    dl = dsv4.DeviceLayer.from_arrays(la)
    q = torch.from_numpy(st.q_idx).cuda()
    w = torch.from_numpy(st.w).cuda()
    pos = torch.from_numpy(st.pos).cuda()
    n_t = torch.tensor([n, 301], dtype=torch.int32, device="cuda")
    idx, scores = dsv4.indexer_topk(q, w, dl.idx_cache, n_t, 64, q_dtype="f32", w_dtype="f32", pos=pos,
                                    q_rope_dims=16)
    torch.cuda.synchronize()
    ol = OA.layer_state(la)
    for s, ns in enumerate([n, 301]):
        qr = O.apply_rope(st.q_idx[s].astype(np.float64), int(st.pos[s]), 16, 1e4)
        ref = O.indexer_scores(qr, st.w[s].astype(np.float64), ol.idx_cache.read(s, np.arange(ns)))
        check_topk(idx[s].cpu().numpy(), ref, 64, ns, f"seq {s}")


# ---------------------------------------------------------------------------- attention
def _mqa_case(spec, B, pos, n_entries, idx=None, seed=41, value_std=1.0, out_dtype=None, garbage_ws=True,
              tweak=None, q_std=None, outlier_frac=0.05):
    la = W.make_layer(spec, B, max(n_entries) + 1, seed, value_std=value_std, outlier_frac=outlier_frac)
    if tweak is not None:
        tweak(la)
    st = W.make_step(spec, B, pos, seed + 1, q_std=value_std if q_std is None else q_std)
    dl = dsv4.DeviceLayer.from_arrays(la)
    q = dsv4.to_device_codes(st.q, spec.q_dtype, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx_t = None if idx is None else torch.from_numpy(idx.astype(np.int32)).cuda()
    args = dict(q_dtype=spec.q_dtype, out_dtype=out_dtype or spec.out_dtype, idx=idx_t,
                n_entries=torch.tensor(n_entries, dtype=torch.int32, device="cuda"), rope_dims=spec.rope_dims)
    ws = None
    if garbage_ws:
        # the workspace holds no state between calls: whatever it contains (NaN bytes here)
        # must not reach the output
        need = dsv4.mqa_workspace_size(dsv4.mqa_args(q, torch.from_numpy(st.pos).cuda(), dl.cache, dl.ring,
                                                             out=torch.empty(1, device="cuda"), **args))
        ws = torch.full((max(need, 256),), 0xFF, dtype=torch.uint8, device="cuda")
    out, lse = dsv4.sparse_mqa_decode(q, torch.from_numpy(st.pos).cuda(), dl.cache, dl.ring, with_lse=True,
                                      d_status=status, workspace=ws, **args)
    torch.cuda.synchronize()
    ol = OA.layer_state(la)
    qd = OA.decode_input(st.q, spec.q_dtype)
    return decode_out(out), lse.cpu().numpy(), status.item(), ol, qd, st


def _ref_attention(ol, qd, st, s, sel, spec, gamma_q=None):
    p = int(st.pos[s])
    parts = [ol.window.read(s, O.window_positions(p, spec.W))]
    if len(sel):
        parts.append(ol.main_cache.read(s, np.asarray(sel)))
    keys = np.concatenate(parts)
    q = qd[s] if gamma_q is None else O.query_norm(qd[s], gamma_q, spec.eps)
    o = O.shared_kv_attention(q, p, keys, 1 / np.sqrt(spec.D), spec.rope_dims, spec.rope_base)
    qr = O.apply_rope(q, p, spec.rope_dims, spec.rope_base)
    lg = qr @ keys.T / np.sqrt(spec.D)
    lse = lg.max(1) + np.log(np.exp(lg - lg.max(1, keepdims=True)).sum(1))
    return o, lse


@pytest.mark.parametrize("out_dtype", ["f32", "bf16"])
def test_mqa_tensor_core_dense_bf16(out_dtype):
    spec = W.C128_SPEC
    pos = [3, 70000, 65536]           # a truncated window, then full ones
    n_entries = [0, 300, 513]          # n_c = 0, then ragged chunk tails
    out, lse, status, ol, qd, st = _mqa_case(spec, 3, pos, n_entries, value_std=1 / np.sqrt(512),
                                             out_dtype=out_dtype)
    assert status == 0
    for s in range(3):
        o, l = _ref_attention(ol, qd, st, s, np.arange(n_entries[s]), spec)
        check_output(out[s], o, "lowp", f"seq {s}", out_dtype=out_dtype)
        assert np.max(np.abs(lse[s] - l)) < 2e-2


def test_mqa_tensor_core_sparse_fp8_with_padding_and_bad_index():
    spec = W.C4_SPEC
    B, n_c = 2, 5000
    rng = np.random.default_rng(5)
    idx = np.stack([rng.permutation(n_c)[:512] for _ in range(B)]).astype(np.int64)
    idx[0, 500:] = -1             # padding
    idx[1, 7] = n_c + 3           # out of range: skipped and reported
    for out_dtype in ("f32", "bf16"):
        out, lse, status, ol, qd, st = _mqa_case(spec, B, [20000, 131072], [n_c, n_c], idx=idx, out_dtype=out_dtype)
        assert status == dsv4._abi.DEV_BAD_INDEX
        for s in range(B):
            sel = [j for j in idx[s] if 0 <= j < n_c]
            o, l = _ref_attention(ol, qd, st, s, sel, spec)
            check_output(out[s], o, "lowp", f"seq {s} out {out_dtype}", out_dtype=out_dtype)
            assert np.max(np.abs(lse[s] - l)) < 2e-2


def test_mqa_tensor_core_rising_logits_rescale_the_output():
    """Selected keys whose logits rise by about 10 (log2 units) from one 64-key chunk to the
    next within each CTA's run: about half of the (head, chunk) steps raise the head's
    reference max by more than the lazy threshold, so the partial output accumulated so far
    is rescaled, chunk after chunk. 40 sequences run two CTAs each (chunks 0-4 and 5-9, the
    first two being the window). The row gains per 64 selected keys keep the largest logit
    near 55 and the outputs of order one, where fp16 operands still meet the tolerance."""
    spec = W.C4_SPEC
    B, n_c = 40, 3000
    gains = [4, 7, 10, 0.3, 3, 6, 9, 1]
    rng = np.random.default_rng(8)
    idx = np.stack([rng.permutation(n_c)[:512] for _ in range(B)]).astype(np.int64)

    def rising(la):
        per_page = spec.per_page
        for s in range(B):
            for u, j in enumerate(idx[s]):
                la.scales[la.block_table[s, j // per_page], j % per_page] *= np.float32(gains[u // 64])

    out, lse, status, ol, qd, st = _mqa_case(spec, B, [131072] * B, [n_c] * B, idx=idx, out_dtype="f32",
                                             tweak=rising, value_std=0.1, q_std=10.0, outlier_frac=0.0)
    assert status == 0
    for s in range(B):
        o, l = _ref_attention(ol, qd, st, s, idx[s], spec)
        check_output(out[s], o, "lowp", f"seq {s}")
        assert np.max(np.abs(lse[s] - l)) < 2e-2


def test_mqa_cuda_core_fp32():
    spec = W.TINY_SPEC
    B = 2
    rng = np.random.default_rng(6)
    idx = np.stack([rng.permutation(1024)[:64] for _ in range(B)]).astype(np.int64)
    idx[1, 60:] = -1
    out, lse, status, ol, qd, st = _mqa_case(spec, B, [4096, 100], [1024, 1024], idx=idx)
    assert status == 0
    for s in range(B):
        sel = [j for j in idx[s] if j >= 0]
        o, l = _ref_attention(ol, qd, st, s, sel, spec)
        check_output(out[s], o, "f32", f"seq {s}")
        assert np.max(np.abs(lse[s] - l)) < 1e-4


@pytest.mark.parametrize("B", [3, 40])  # clusters of 4 CTAs (one 128-column block each) and of 2 (two)
def test_mqa_tensor_core_query_norm_fp8_output(B):
    """Query norm before RoPE and fp8 output in 128-channel blocks, fused in the attention's
    query preparation and merge epilogue."""
    spec = W.C4_SPEC
    n_c = 3000
    rng = np.random.default_rng(9)
    idx = np.stack([rng.permutation(n_c)[:512] for _ in range(B)]).astype(np.int64)
    la = W.make_layer(spec, B, n_c + 1, 43, outlier_frac=0.05)
    st = W.make_step(spec, B, [131072 - 7 * i for i in range(B)], 44, q_std=3.0)
    gq = (1.0 + 0.2 * rng.standard_normal(spec.D)).astype(np.float32)
    dl = dsv4.DeviceLayer.from_arrays(la)
    q = dsv4.to_device_codes(st.q, spec.q_dtype, "cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    (codes, scales) = dsv4.sparse_mqa_decode(
        q, torch.from_numpy(st.pos).cuda(), dl.cache, dl.ring, q_dtype=spec.q_dtype, out_dtype="fp8",
        idx=torch.from_numpy(idx.astype(np.int32)).cuda(), n_entries=torch.full((B,), n_c, dtype=torch.int32,
                                                                                device="cuda"),
        rope_dims=spec.rope_dims, d_status=status, q_norm_gamma=torch.from_numpy(gq).cuda(), q_norm_eps=spec.eps)
    torch.cuda.synchronize()
    assert status.item() == 0
    ol = OA.layer_state(la)
    qd = OA.decode_input(st.q, spec.q_dtype)
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    for s_ in range(B):
        o, _ = _ref_attention(ol, qd, st, s_, idx[s_], spec, gamma_q=gq.astype(np.float64))
        check_output_fp8(codes[s_], scales[s_], o, "lowp", f"seq {s_}")


def test_mqa_cuda_core_query_norm_fp8_output():
    spec = W.TINY_SPEC
    B = 2
    rng = np.random.default_rng(10)
    idx = np.stack([rng.permutation(1024)[:64] for _ in range(B)]).astype(np.int64)
    la = W.make_layer(spec, B, 1025, 45)
    st = W.make_step(spec, B, [4096, 300], 46)
    gq = (1.0 + 0.2 * rng.standard_normal(spec.D)).astype(np.float32)
    dl = dsv4.DeviceLayer.from_arrays(la)
    (codes, scales) = dsv4.sparse_mqa_decode(
        torch.from_numpy(st.q).cuda(), torch.from_numpy(st.pos).cuda(), dl.cache, dl.ring, q_dtype="f32",
        out_dtype="fp8", idx=torch.from_numpy(idx.astype(np.int32)).cuda(),
        n_entries=torch.full((B,), 1024, dtype=torch.int32, device="cuda"), rope_dims=spec.rope_dims,
        q_norm_gamma=torch.from_numpy(gq).cuda(), q_norm_eps=spec.eps)
    torch.cuda.synchronize()
    ol = OA.layer_state(la)
    qd = OA.decode_input(st.q, spec.q_dtype)
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    for s_ in range(B):
        o, _ = _ref_attention(ol, qd, st, s_, idx[s_], spec, gamma_q=gq.astype(np.float64))
        check_output_fp8(codes[s_], scales[s_], o, "f32", f"seq {s_}")
