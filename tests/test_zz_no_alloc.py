"""dsv4_indexer_topk_noalloc: the indexer top-k on the library's static scratch.

The host-side test needs no GPU: a request larger than the scratch is refused with
DSV4_ERR_SCRATCH_LIMIT before anything launches. The GPU test calls the no-alloc entry
point twice in a row through the C ABI and compares each result with the workspace entry
point on the same inputs (indices exactly, scores exactly: both run the same kernels).
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


def _inputs(n_list, seed=31):
    spec = W.C4_SPEC
    B = len(n_list)
    la = W.make_layer(spec, B, max(n_list) + 1, seed, outlier_frac=0.05)
    st = W.make_step(spec, B, 0, seed + 1)
    dl = dsv4.DeviceLayer.from_arrays(la)
    q = dsv4.to_device_codes(st.q_idx, spec.q_idx_dtype, "cuda")
    w = dsv4.to_device_codes(st.w, spec.w_dtype, "cuda")
    n = torch.tensor(n_list, dtype=torch.int32, device="cuda")
    qs = torch.from_numpy(st.q_idx_scale).cuda()
    return spec, dl, q, w, n, qs


def _sorted_pairs(idx, scores):
    idx = idx.cpu().numpy()
    scores = scores.cpu().numpy()
    order = np.argsort(idx, axis=1, kind="stable")
    return np.take_along_axis(idx, order, 1), np.take_along_axis(scores, order, 1)


@pytest.mark.gpu
@pytest.mark.parametrize("k", [512, 1024])  # tensor-core path, CUDA-core path
def test_noalloc_matches_workspace_entry_point_twice(k):
    require_gpu()
    n_list = [130, 5000, 20000, 0, 777]
    spec, dl, q, w, n, qs = _inputs(n_list)
    common = dict(q_dtype=spec.q_idx_dtype, w_dtype=spec.w_dtype, q_scale=qs)
    a = dsv4.indexer_args(q, w, dl.idx_cache, n, k, **common)
    assert dsv4.load().dsv4_indexer_workspace_size(C.byref(a)) <= A.NOALLOC_SCRATCH_BYTES
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
