"""Host-side checks of the C ABI that need no GPU.

The library loads, exports every function include/dsv4.h declares, its host
helpers answer, and argument validation rejects bad calls synchronously before
any launch (so these calls are safe on a machine without a device).
"""

import ctypes as C
import json
import os
import re

import pytest

import compressed_sparse_kv_dsv4_b200 as dsv4
from compressed_sparse_kv_dsv4_b200 import _abi as A
import oracle.dsv4_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000  # a 16-byte-aligned dummy address; validation never dereferences pointers


@pytest.fixture(scope="module")
def lib():
    return dsv4.load()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "dsv4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsv4_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_function_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(lib, n), n
        assert n in A.EXPORTS, f"{n} has no binding"


def test_package_exports_every_binding_call():
    """Each public function and class of the binding is reachable from the package."""
    import inspect

    from compressed_sparse_kv_dsv4_b200 import binding

    names = [n for n, v in vars(binding).items() if not n.startswith("_") and (inspect.isfunction(v) or
             inspect.isclass(v)) and getattr(v, "__module__", "") == binding.__name__]
    assert "indexer_scores" in names
    missing = [n for n in names if not hasattr(dsv4, n)]
    assert not missing, missing


def test_host_helpers(lib, golden_dir):
    assert lib.dsv4_abi_version() == 3
    assert lib.dsv4_status_string(A.OK) == b"ok"
    assert lib.dsv4_status_string(A.ERR_INVALID_ARG) == b"invalid argument"
    assert lib.dsv4_status_string(99) == b"unknown status"
    g = json.load(open(os.path.join(golden_dir, "kv_state_sizing.json")))
    L = g["context_tokens"]
    gib = float(1 << 30)
    v4 = (30 * lib.dsv4_layer_state_bytes(L, 4, 640, 0, 0, 2) + 31 * lib.dsv4_layer_state_bytes(L, 128, 512, 0, 0, 2))
    v32 = 61 * lib.dsv4_layer_state_bytes(L, 1, 704, 0, 0, 2)
    assert round(v4 / gib, 2) == g["v4_gib"] and round(v32 / gib, 1) == g["v32_gib"]
    # same closed form as the oracle's, with a window
    for m, ew, w, ww in ((4, 640, 128, 512), (128, 512, 128, 512), (1, 100, 0, 0)):
        assert lib.dsv4_layer_state_bytes(123457, m, ew, w, ww, 2) == O.kv_state_bytes(123457, [(m, ew, w, ww)], 2)
    assert lib.dsv4_layer_state_bytes(10, 0, 1, 0, 0, 2) == 0


def _cache(dim=512, m=4, dtype=A.FP8, scales=FAKE):
    return A.PagedCache(FAKE, scales, FAKE, 64, 8, dim, m, dtype)


def _ring(dim=512, dtype=A.FP8):
    return A.WindowRing(FAKE, FAKE, 128, dim, dtype)


def _mqa(**kw):
    a = A.MqaArgs(batch=2, heads=64, dim=512, q=FAKE, q_dtype=A.BF16, pos=FAKE, cache=_cache(), n_entries=FAKE,
                  idx=None, k=0, ring=_ring(), softmax_scale=0.0, rope=A.Rope(64, 1e4), out=FAKE, out_dtype=A.BF16,
                  lse=None, d_status=None)
    for k_, v in kw.items():
        setattr(a, k_, v)
    return a


def _indexer(**kw):
    a = A.IndexerArgs(batch=2, heads=64, dim=128, k=512, q_idx=FAKE, q_dtype=A.FP8, q_scale=FAKE, w=FAKE,
                      w_dtype=A.BF16, keys=_cache(dim=128), n_entries=FAKE, pos=None, q_rope_dims=0, rope_base=1e4,
                      idx=FAKE, scores=None, d_status=None)
    for k_, v in kw.items():
        setattr(a, k_, v)
    return a


def test_attention_workspace_covers_the_cluster_exchange(lib):
    """The tensor-core attention splits each sequence over a cluster of cs CTAs (a power of
    two up to 16 that keeps the batch within one wave of the 148 SMs) whose partial outputs,
    (cs - 1) slabs of [64 heads][512 / cs] fp32 per CTA, pass through the workspace; the
    prepared query (bf16/fp16, [B][64][512]) sits there too. No GPU here: 148 SMs assumed."""
    for batch, cs in ((1, 16), (2, 16), (9, 16), (10, 8), (32, 4), (37, 4), (40, 2), (74, 2), (75, 1)):
        a = _mqa(batch=batch)
        need = lib.dsv4_mqa_workspace_size(C.byref(a))
        partials = batch * (cs - 1) * 64 * 512 * 4
        query = batch * 64 * 512 * 2
        assert need >= partials + query, (batch, need)
        # nothing else of size: per-sequence scales and (max, sum) pairs, and alignment
        assert need - partials - query <= batch * (64 * 4 + 16 * 2 * 64 * 4) + 3 * 256, (batch, need)


def test_validation_rejects_bad_calls(lib):
    # null argument structs
    assert lib.dsv4_compress(None, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_swa_insert(None, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_indexer_topk(None, None, 0, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_sparse_mqa_decode(None, None, 0, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_hybrid_decode(None, None, None, 0, None) == A.ERR_INVALID_ARG
    # attention: bad shapes / pointers / dtypes
    for bad, code in ((dict(batch=0), A.ERR_INVALID_ARG), (dict(q=None), A.ERR_INVALID_ARG),
                      (dict(q=FAKE + 4), A.ERR_INVALID_ARG), (dict(dim=500), A.ERR_INVALID_ARG),
                      (dict(q_dtype=A.FP8), A.ERR_UNSUPPORTED), (dict(out_dtype=A.FP8), A.ERR_INVALID_ARG),
                      (dict(out_dtype=7), A.ERR_UNSUPPORTED),
                      (dict(q_norm_gamma=FAKE, q_norm_eps=-1.0), A.ERR_INVALID_ARG),
                      (dict(rope=A.Rope(63, 1e4)), A.ERR_INVALID_ARG), (dict(n_entries=None), A.ERR_INVALID_ARG),
                      (dict(cache=_cache(scales=None)), A.ERR_INVALID_ARG),
                      (dict(cache=_cache(m=3)), A.ERR_INVALID_ARG),
                      (dict(ring=_ring(dtype=A.BF16)), A.ERR_INVALID_ARG)):
        a = _mqa(**bad)
        assert lib.dsv4_sparse_mqa_decode(C.byref(a), C.c_void_p(FAKE), 1 << 30, None) == code, bad
        assert lib.dsv4_mqa_workspace_size(C.byref(a)) == 0
    # fp8 output with its block scales, and a query norm, are accepted
    assert lib.dsv4_mqa_workspace_size(C.byref(_mqa(out_dtype=A.FP8, out_scales=FAKE))) > 0
    assert lib.dsv4_mqa_workspace_size(C.byref(_mqa(q_norm_gamma=FAKE, q_norm_eps=1e-6))) > 0
    # a too-small workspace is rejected before any launch
    a = _mqa()
    need = lib.dsv4_mqa_workspace_size(C.byref(a))
    assert need > 0
    assert lib.dsv4_sparse_mqa_decode(C.byref(a), C.c_void_p(FAKE), need - 1, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_sparse_mqa_decode(C.byref(a), C.c_void_p(FAKE + 16), need, None) == A.ERR_INVALID_ARG
    # indexer scores alone: the tensor-core shapes, an aligned output with a wide enough stride
    ia = _indexer()
    cap = ia.keys.max_blocks * (256 // ia.keys.m)
    assert lib.dsv4_indexer_scores(None, C.c_void_p(FAKE), cap, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_indexer_scores(C.byref(ia), None, cap, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_indexer_scores(C.byref(ia), C.c_void_p(FAKE + 4), cap, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_indexer_scores(C.byref(ia), C.c_void_p(FAKE), cap - 4, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_indexer_scores(C.byref(_indexer(q_dtype=A.F32)), C.c_void_p(FAKE), cap, None) == A.ERR_UNSUPPORTED
    # indexer
    for bad, code in ((dict(k=0), A.ERR_INVALID_ARG), (dict(idx=None), A.ERR_INVALID_ARG),
                      (dict(dim=64), A.ERR_INVALID_ARG), (dict(q_dtype=A.BF16), A.ERR_UNSUPPORTED),
                      (dict(keys=_cache(dim=128, dtype=A.BF16)), A.ERR_UNSUPPORTED),
                      (dict(q_rope_dims=16), A.ERR_INVALID_ARG), (dict(k=4096), A.ERR_UNSUPPORTED)):
        a = _indexer(**bad)
        assert lib.dsv4_indexer_topk(C.byref(a), C.c_void_p(FAKE), 1 << 30, None) == code, bad
    # fp4 (e2m1) keys: accepted for the indexer with their scales, never as an attention cache
    assert lib.dsv4_indexer_workspace_size(C.byref(_indexer(keys=_cache(dim=128, dtype=A.FP4)))) > 0
    assert lib.dsv4_indexer_workspace_size(C.byref(_indexer(keys=_cache(dim=128, dtype=A.FP4, scales=None)))) == 0
    assert lib.dsv4_mqa_workspace_size(C.byref(_mqa(cache=_cache(dtype=A.FP4)))) == 0
    a = _indexer()
    need = lib.dsv4_indexer_workspace_size(C.byref(a))
    assert need >= 2 * 512 * 4  # at least one float score per cache entry of each sequence
    assert lib.dsv4_indexer_topk(C.byref(a), C.c_void_p(FAKE), need - 1, None) == A.ERR_INVALID_ARG


def test_compress_and_window_validation(lib):
    state = A.CompressorState(FAKE, 4, 512, 512)
    a = A.CompressArgs(batch=2, total_tokens=10, kv=FAKE, gate=FAKE, kv_dtype=A.BF16, cu_seqlens=FAKE,
                       start_pos=FAKE, gamma=FAKE, eps=1e-6, rope=A.Rope(64, 1e4), state=state, cache=_cache(),
                       d_status=None)
    for field, val, code in (("kv_dtype", A.FP8, A.ERR_UNSUPPORTED), ("batch", 0, A.ERR_INVALID_ARG),
                             ("gamma", None, A.ERR_INVALID_ARG), ("eps", -1.0, A.ERR_INVALID_ARG)):
        b = A.CompressArgs.from_buffer_copy(a)
        setattr(b, field, val)
        assert lib.dsv4_compress(C.byref(b), None) == code, field
    b = A.CompressArgs.from_buffer_copy(a)
    b.state = A.CompressorState(FAKE, 8, 512, 512)  # state rate differs from the cache's
    assert lib.dsv4_compress(C.byref(b), None) == A.ERR_INVALID_ARG
    b.state = A.CompressorState(FAKE, 4, 512, 7)  # gate width must be 1 or dim
    assert lib.dsv4_compress(C.byref(b), None) == A.ERR_INVALID_ARG
    b = A.CompressArgs.from_buffer_copy(a)
    b.total_tokens = 0  # nothing to do
    assert lib.dsv4_compress(C.byref(b), None) == A.OK
    w = A.SwaInsertArgs(batch=1, total_tokens=3, kv=FAKE, kv_dtype=A.F32, cu_seqlens=FAKE, start_pos=FAKE,
                        gamma=FAKE, eps=1e-6, rope=A.Rope(64, 1e4), ring=_ring(dtype=A.FP8, dim=512), d_status=None)
    w2 = A.SwaInsertArgs.from_buffer_copy(w)
    w2.ring = A.WindowRing(FAKE, None, 128, 512, A.FP8)  # fp8 ring without scales
    assert lib.dsv4_swa_insert(C.byref(w2), None) == A.ERR_INVALID_ARG
    w2 = A.SwaInsertArgs.from_buffer_copy(w)
    w2.total_tokens = 0
    assert lib.dsv4_swa_insert(C.byref(w2), None) == A.OK


def test_compress_project_validation_and_workspace(lib):
    """dsv4_compress_project: the compressor's checks, plus hidden_dim % 64, dim % 128 and one
    gate per channel; the workspace holds the projected kv and gate (bf16, 256-byte aligned)."""
    state = A.CompressorState(FAKE, 4, 512, 512)
    c = A.CompressArgs(batch=2, total_tokens=1000, kv=None, gate=None, kv_dtype=A.F32, cu_seqlens=FAKE,
                       start_pos=FAKE, gamma=FAKE, eps=1e-6, rope=A.Rope(64, 1e4), state=state, cache=_cache(),
                       d_status=None)
    a = A.CompressProjectArgs(c=c, hidden=FAKE, w=FAKE, hidden_dim=4096)
    need = lib.dsv4_compress_project_workspace_size(C.byref(a))
    per = (1000 * 512 * 2 + 255) // 256 * 256
    assert 2 * per <= need <= 2 * per + 256
    assert lib.dsv4_compress_project(None, None, 0, None) == A.ERR_INVALID_ARG
    for field, val, code in (("hidden_dim", 100, A.ERR_UNSUPPORTED), ("hidden_dim", 0, A.ERR_INVALID_ARG),
                             ("hidden", None, A.ERR_INVALID_ARG), ("w", FAKE + 8, A.ERR_INVALID_ARG)):
        b = A.CompressProjectArgs.from_buffer_copy(a)
        setattr(b, field, val)
        assert lib.dsv4_compress_project(C.byref(b), C.c_void_p(FAKE), need, None) == code, field
        assert lib.dsv4_compress_project_workspace_size(C.byref(b)) == 0
    b = A.CompressProjectArgs.from_buffer_copy(a)
    b.c.state = A.CompressorState(FAKE, 4, 512, 1)  # one gate per token: not what the projection makes
    assert lib.dsv4_compress_project(C.byref(b), C.c_void_p(FAKE), need, None) == A.ERR_UNSUPPORTED
    b = A.CompressProjectArgs.from_buffer_copy(a)
    b.c.state = A.CompressorState(FAKE, 4, 192, 192)
    b.c.cache = _cache(dim=192)
    assert lib.dsv4_compress_project(C.byref(b), C.c_void_p(FAKE), 1 << 30, None) == A.ERR_UNSUPPORTED
    # a short or misaligned workspace is refused before any launch
    assert lib.dsv4_compress_project(C.byref(a), C.c_void_p(FAKE), need - 1, None) == A.ERR_INVALID_ARG
    assert lib.dsv4_compress_project(C.byref(a), C.c_void_p(FAKE + 16), need, None) == A.ERR_INVALID_ARG
    b = A.CompressProjectArgs.from_buffer_copy(a)
    b.c.total_tokens = 0  # nothing to do
    assert lib.dsv4_compress_project(C.byref(b), None, 0, None) == A.OK


def test_hybrid_validation_and_workspace(lib):
    L = A.Layer()
    L.kind, L.heads, L.dim, L.topk, L.idx_heads, L.idx_dim = A.LAYER_C4, 64, 512, 512, 64, 128
    L.rope = A.Rope(64, 1e4)
    L.idx_rope_dims, L.eps = 64, 1e-6
    L.gamma, L.gamma_idx = FAKE, FAKE
    L.state = A.CompressorState(FAKE, 4, 512, 512)
    L.cache = _cache()
    L.ring = _ring()
    L.idx_state = A.CompressorState(FAKE, 4, 128, 128)
    L.idx_cache = _cache(dim=128)
    ws = lib.dsv4_hybrid_decode_workspace_size(C.byref(L), 32)
    assert ws >= 32 * 512 * 4
    L2 = A.Layer.from_buffer_copy(L)
    L2.idx_state = A.CompressorState(FAKE, 8, 128, 128)
    assert lib.dsv4_hybrid_decode_workspace_size(C.byref(L2), 32) == 0
    L2 = A.Layer.from_buffer_copy(L)
    L2.kind = 7
    assert lib.dsv4_hybrid_decode_workspace_size(C.byref(L2), 32) == 0
    S = A.Step()
    S.batch, S.pos, S.kv, S.gate, S.q, S.out = 32, FAKE, FAKE, FAKE, FAKE, FAKE
    S.kv_dtype, S.q_dtype, S.out_dtype = A.BF16, A.BF16, A.BF16
    S.idx_kv, S.idx_gate, S.q_idx, S.w = FAKE, FAKE, FAKE, FAKE
    S.q_idx_dtype, S.w_dtype = A.FP8, A.BF16
    # the layer-level size is the largest need over the step's dtype choices; a workspace
    # below one score per cache entry of every sequence is too small for any of them
    assert lib.dsv4_hybrid_decode(C.byref(L), C.byref(S), C.c_void_p(FAKE), 32 * 512 * 4 - 1, None) == A.ERR_INVALID_ARG
    S2 = A.Step.from_buffer_copy(S)
    S2.batch = 31  # disagrees with nothing yet, but a missing q must be caught
    S2.q = None
    assert lib.dsv4_hybrid_decode(C.byref(L), C.byref(S2), C.c_void_p(FAKE), ws, None) == A.ERR_INVALID_ARG
    S2 = A.Step.from_buffer_copy(S)
    S2.q_idx_dtype = A.BF16
    assert lib.dsv4_hybrid_decode(C.byref(L), C.byref(S2), C.c_void_p(FAKE), ws, None) == A.ERR_UNSUPPORTED
