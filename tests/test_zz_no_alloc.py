"""dsv4_indexer_topk_noalloc: the indexer top-k on the library's static scratch.

The host-side test needs no GPU: a request larger than the scratch is refused with
DSV4_ERR_SCRATCH_LIMIT before anything launches. The GPU test calls the no-alloc entry
point twice in a row through the C ABI, on the tensor-core and on the CUDA-core path, and
compares each result with the workspace entry point on the same inputs (indices exactly,
scores exactly: both run the same kernels).
This file sorts last so that the GPU test also runs after every other test has used the
device.
"""

import ctypes as C

import numpy as np
import pytest
import torch

import compressed_sparse_kv_dsv4_b200 as dsv4
from compressed_sparse_kv_dsv4_b200 import _abi as A
import synthetic as W
from tests.parity import require_gpu

FAKE = 0x10000  # a 16-byte-aligned dummy address; validation never dereferences pointers


def _args(batch, max_blocks, k=512):
    keys = A.PagedCache(FAKE, FAKE, FAKE, 64, max_blocks, 128, 4, A.FP8)
    return A.IndexerArgs(batch=batch, heads=64, dim=128, k=k, q_idx=FAKE, q_dtype=A.FP8, q_scale=FAKE, w=FAKE,
                         w_dtype=A.BF16, keys=keys, n_entries=FAKE, pos=None, q_rope_dims=0, rope_base=1e4,
                         idx=FAKE, scores=None, d_status=None)


def test_noalloc_refuses_requests_beyond_the_scratch():
    lib = dsv4.load()
    big = _args(batch=160, max_blocks=512)  # 131072 positions: 32768 entries per sequence
    assert lib.dsv4_indexer_workspace_size(C.byref(big)) > A.NOALLOC_SCRATCH_BYTES
    assert lib.dsv4_indexer_topk_noalloc(C.byref(big), None) == A.ERR_SCRATCH_LIMIT
    assert b"static scratch" in lib.dsv4_status_string(A.ERR_SCRATCH_LIMIT)
    assert lib.dsv4_indexer_topk_noalloc(None, None) == A.ERR_INVALID_ARG


def _inputs(n_list, q_dtype, seed=31):
    spec = W.C4_SPEC
    B = len(n_list)
    la = W.make_layer(spec, B, max(n_list) + 1, seed, outlier_frac=0.05)
    st = W.make_step(spec, B, 0, seed + 1)
    dl = dsv4.DeviceLayer.from_arrays(la)
    w = dsv4.to_device_codes(st.w, spec.w_dtype, "cuda")
    n = torch.tensor(n_list, dtype=torch.int32, device="cuda")
    if q_dtype == "fp8":
        q = dsv4.to_device_codes(st.q_idx, "fp8", "cuda")
        qs = torch.from_numpy(st.q_idx_scale).cuda()
    else:  # the same query values as float32 (exact: e4m3 code times a power-of-two scale)
        vals = torch.from_numpy(st.q_idx.copy()).view(torch.float8_e4m3fn).float().numpy()
        q = torch.from_numpy((vals * st.q_idx_scale[..., None]).astype(np.float32)).cuda()
        qs = None
    return spec, dl, q, w, n, qs


def _sorted_pairs(idx, scores):
    idx = idx.cpu().numpy()
    scores = scores.cpu().numpy()
    order = np.argsort(idx, axis=1, kind="stable")
    return np.take_along_axis(idx, order, 1), np.take_along_axis(scores, order, 1)


@pytest.mark.gpu
@pytest.mark.parametrize("k,q_dtype,tensor_cores", [(512, "fp8", True), (1024, "fp8", True), (512, "f32", False)])
def test_noalloc_matches_workspace_entry_point_twice(k, q_dtype, tensor_cores):
    """fp8 queries take the tensor-core path (scores streamed to the scratch, then the cluster
    top-k); float32 queries take the CUDA-core path (candidate counts zeroed at the head of the
    scratch, then a candidate list per sequence)."""
    require_gpu()
    n_list = [130, 5000, 20000, 0, 777]
    spec, dl, q, w, n, qs = _inputs(n_list, q_dtype)
    common = dict(q_dtype=q_dtype, w_dtype=spec.w_dtype, q_scale=qs)
    probe = torch.empty((len(n_list), k), dtype=torch.int32, device="cuda")
    a = dsv4.indexer_args(q, w, dl.idx_cache, n, k, idx=probe, **common)
    need = dsv4.load().dsv4_indexer_workspace_size(C.byref(a))
    assert 0 < need <= A.NOALLOC_SCRATCH_BYTES
    # the CUDA-core path keeps a 64-bit candidate per cache entry of every sequence
    cand_bytes = len(n_list) * dl.idx_cache.block_table.shape[1] * 64 * 8
    assert (need >= cand_bytes) == (not tensor_cores)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    ref_idx, ref_scores = dsv4.indexer_topk(q, w, dl.idx_cache, n, k, d_status=status, **common)
    want = _sorted_pairs(ref_idx, ref_scores)
    B = len(n_list)
    for call in range(2):
        idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
        scores = torch.full((B, k), 7.0, dtype=torch.float32, device="cuda")
        dsv4.indexer_topk_noalloc(q, w, dl.idx_cache, n, k, idx=idx, scores=scores, d_status=status, **common)
        torch.cuda.synchronize()
        assert status.item() == 0
        got = _sorted_pairs(idx, scores)
        assert np.array_equal(got[0], want[0]), f"call {call}: indices differ"
        assert np.array_equal(got[1], want[1]), f"call {call}: scores differ"
