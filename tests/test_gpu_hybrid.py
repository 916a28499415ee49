"""GPU parity of dsv4_hybrid_decode on the benchmark workloads, against the oracle.

  tiny C4, fp32     built end to end from hidden states (prefill through the GPU's own
                    compressor and window insert on one side, the oracle's on the other),
                    then one decode step at position 4096.
  C128 dense, bf16  B = 8, 65536-token context.
  C4 sparse, fp8    B = 32, 131072-token context (the benchmark's launch configuration),
                    five steps; at the step that completes a block, eight sequences get a new
                    indexer entry built to rank among their top k, so a read of that entry
                    before the step's own append is caught.
  1M stack          two C4 + two C128 layers, B = 4, 16 consecutive decode steps; the oracle
                    follows every state update and checks the attention at steps 0, 3 and 15.
  first tokens      a C4 step where no sequence has a complete block yet (positions 0..2):
                    no indexer tile at all, the attention reads only the window the step's
                    own prologue has just written.

Every step's own writes (the window slot, the compressor state rings, each appended main and
indexer entry) are compared with the oracle's, and the top-k sets must match the oracle's
exactly (near ties aside): only an appended entry whose stored bytes are shown to differ
between the two sides may swap. Outputs are checked once stored as float32 (the bounds as
written) and once as bf16 (against the oracle's output rounded to bf16).
"""

import dataclasses

import numpy as np
import pytest
import torch

import compressed_sparse_kv_dsv4_b200 as dsv4
import oracle.dsv4_oracle as O
import synthetic as W
from oracle import adapters as OA
from tests.parity import (check_output, check_output_fp8, check_step_writes, check_topk, codes_close, decode_out,
                          input_class, require_gpu)

pytestmark = pytest.mark.gpu

OUT_DTYPES = ["f32", "bf16"]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _with_out(spec, out_dtype):
    return dataclasses.replace(spec, out_dtype=out_dtype)


def _step_and_check(dl, ol, spec, st, seqs=None, attend=True, must_select=None):
    """One decode step on both sides; checks the step's writes and (attend) the outputs.
    must_select: {seq: entry} that the oracle's own top k must contain (a check of how the
    test built its inputs)."""
    ds = dsv4.DeviceStep.from_arrays(spec, st)
    dsv4.hybrid_decode(dl, ds)
    torch.cuda.synchronize()
    assert ds.d_status.item() == 0, f"device status {ds.d_status.item()}"
    oin = OA.step_inputs(spec, st)
    O.decode_update(ol, oin)
    differ = check_step_writes(dl, ol, spec, st)
    if not attend:
        return 0, differ
    res = O.decode_attend(ol, oin, seqs)
    out = ds.out.cpu().numpy() if spec.out_dtype == "fp8" else decode_out(ds.out)
    idx = ds.topk_idx.cpu().numpy() if ds.topk_idx is not None else None
    swaps = 0
    for s, (o, sel, scores) in res.items():
        if spec.kind == "c4":
            n_c = O.visible_entries(int(st.pos[s]), spec.m)
            if must_select and s in must_select:
                assert must_select[s] in set(sel.tolist()), f"seq {s}: test input did not rank the new entry"
                if must_select[s] not in differ[s]:
                    assert must_select[s] in set(idx[s].tolist()), f"seq {s}: new entry {must_select[s]} not selected"
            swaps += check_topk(idx[s], scores, spec.k, n_c, f"seq {s}", excused=differ[s])
        if spec.out_dtype == "fp8":
            check_output_fp8(out[s], ds.out_scales[s].cpu().numpy(), o, input_class(spec), f"seq {s}")
        else:
            check_output(out[s], o, input_class(spec), f"seq {s}", out_dtype=spec.out_dtype)
    return swaps, differ


def _rank_new_index_entry(spec, st, s, ol):
    """Rewrite sequence s's new indexer token so that the entry its block completes ranks
    high: its gate (+30 in every channel) outweighs the block's three earlier tokens, and its
    kv points along sum_h w_h q_h, rotated back by the entry's RoPE so that the stored key
    (after RMSNorm and RoPE at the block position) points that way."""
    p = int(st.pos[s])
    assert (p + 1) % spec.m == 0
    q = OA.decode_input(st.q_idx, spec.q_idx_dtype, st.q_idx_scale)[s]
    w = OA.decode_input(st.w, spec.w_dtype)[s]
    v = (w[:, None] * q).sum(0)
    v = v / np.sqrt(np.mean(v * v))
    v = O.apply_rope(v, (p // spec.m) * spec.m, spec.idx_rope_dims, spec.rope_base, inverse=True)
    st.idx_kv[s] = W.encode_values(v.astype(np.float32), spec.kv_dtype)
    st.idx_gate[s] = W.encode_values(np.full(spec.d_I, 30.0, np.float32), spec.kv_dtype)
    return p // spec.m


def test_tiny_c4_fp32_end_to_end():
    wl = W.tiny_c4_fp32()
    spec = wl.layer.spec
    L = wl.prefix_kv.shape[0]
    dl = dsv4.DeviceLayer.from_arrays(wl.layer)
    ol = OA.layer_state(wl.layer)
    cu = torch.tensor([0, L], dtype=torch.int32, device="cuda")
    sp = torch.tensor([0], dtype=torch.int32, device="cuda")
    f = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dsv4.compress(f(wl.prefix_kv), f(wl.prefix_gate), cu, sp, dl.state, dl.cache, dl.gamma, kv_dtype="f32",
                  rope_dims=spec.rope_dims, d_status=status)
    dsv4.compress(f(wl.prefix_idx_kv), f(wl.prefix_idx_gate), cu, sp, dl.idx_state, dl.idx_cache, dl.gamma_idx,
                  kv_dtype="f32", rope_dims=spec.idx_rope_dims, d_status=status)
    dsv4.swa_insert(f(wl.prefix_kv), cu, sp, dl.ring, dl.gamma, kv_dtype="f32", rope_dims=spec.rope_dims,
                    d_status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    kv = wl.prefix_kv.astype(np.float64)
    O.compress(kv, wl.prefix_gate.astype(np.float64), [0, L], [0], ol.main_state, ol.main_cache, ol.gamma,
               spec.eps, spec.rope_dims, spec.rope_base)
    O.compress(wl.prefix_idx_kv.astype(np.float64), wl.prefix_idx_gate.astype(np.float64), [0, L], [0],
               ol.idx_state, ol.idx_cache, ol.gamma_idx, spec.eps, spec.idx_rope_dims, spec.rope_base)
    for t in range(L - spec.W, L):
        O.swa_insert(ol.window, 0, t, kv[t], ol.gamma, spec.eps, spec.rope_dims, spec.rope_base)
    # the prefix the two compressors built: float32 rows equal up to float32 rounding
    pages = dsv4.to_numpy_codes(dl.cache.pages, spec.cache_dtype)
    ipages = dsv4.to_numpy_codes(dl.idx_cache.pages, spec.idx_dtype)
    for j in range(L // spec.m):
        pg, sl = ol.main_cache.locate(0, j)
        codes_close(pages[pg, sl], ol.main_cache.pages[pg, sl], 1.0, 1.0, "f32", f"prefix entry {j}")
        pg, sl = ol.idx_cache.locate(0, j)
        codes_close(ipages[pg, sl], ol.idx_cache.pages[pg, sl], 1.0, 1.0, "f32", f"prefix indexer entry {j}")
    # the indexer reads float32 keys that may differ in the last bit: a swap must be a near tie
    # of the oracle's scores (the rule above, with no entry excused)
    swaps, _ = _step_and_check(dl, ol, spec, wl.step)
    assert swaps <= 2


@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
def test_c128_dense_bf16_full_size(out_dtype):
    la, steps = W.c128_dense_bf16()
    spec = _with_out(la.spec, out_dtype)
    dl = dsv4.DeviceLayer.from_arrays(la)
    ol = OA.layer_state(la)
    _step_and_check(dl, ol, spec, steps[0])


@pytest.mark.slow
@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
def test_c4_sparse_131k_full_size(out_dtype):
    la, steps = W.c4_sparse(steps=5)
    spec = _with_out(la.spec, out_dtype)
    dl = dsv4.DeviceLayer.from_arrays(la)
    ol = OA.layer_state(la)
    # five consecutive steps: positions 131072..131076; the block of 131072..131075 completes
    # at step 3, where sequences 0..7 get a new indexer entry built to rank in their top k
    for i, st in enumerate(steps):
        attend = i in (0, 3, 4)
        must = None
        if i == 3:
            must = {s: _rank_new_index_entry(spec, st, s, ol) for s in range(8)}
        _step_and_check(dl, ol, spec, st, seqs=range(la.B) if attend else None, attend=attend, must_select=must)


@pytest.mark.slow
@pytest.mark.parametrize("out_dtype", OUT_DTYPES)
def test_stack_1m_sixteen_steps(out_dtype):
    layers, step_sets = W.stack_1m(steps=16)
    dls = [dsv4.DeviceLayer.from_arrays(la) for la in layers]
    ols = [OA.layer_state(la) for la in layers]
    for i in range(16):
        for li, la in enumerate(layers):
            spec = _with_out(la.spec, out_dtype)
            attend = i in (0, 3, 15)
            must = None
            if spec.kind == "c4" and i == 3:  # the first new C4 entry of the run
                must = {s: _rank_new_index_entry(spec, step_sets[li][i], s, ols[li]) for s in (0, 2)}
            _step_and_check(dls[li], ols[li], spec, step_sets[li][i], attend=attend, must_select=must)


@pytest.mark.parametrize("out_dtype,idx_dtype", [("f32", "fp8"), ("bf16", "fp8"), ("bf16", "fp4")])
def test_c4_first_tokens_window_only(out_dtype, idx_dtype):
    """Positions 0, 1, 2 (then one step further): no complete block in any sequence at the
    first step, so the indexer has no tile; the output is the window-only softmax over the
    positions 0..p, the newest of which the step itself inserted.

    The window and the main cache are bf16 here (the indexer stays fp8 or fp4, on the tensor cores):
    with one to three keys the output is nearly the new key itself, and an fp8 code that the
    two sides round one step apart (allowed for rows each side builds itself) would move it
    by up to 1/16 of the element, more than the output bound; one bf16 step stays within it."""
    spec = _with_out(dataclasses.replace(W.C4_SPEC, cache_dtype="bf16", swa_dtype="bf16", idx_dtype=idx_dtype),
                     out_dtype)
    B = 3
    la = W.make_layer(spec, B, 4, seed=61, outlier_frac=0.05)
    dl = dsv4.DeviceLayer.from_arrays(la)
    ol = OA.layer_state(la)
    for i in range(3):
        st = W.make_step(spec, B, [0 + i, 1 + i, 2 + i], seed=62 + i)
        _step_and_check(dl, ol, spec, st)


@pytest.mark.parametrize("kind", ["c4", "c128"])
def test_query_norm_and_fp8_output_step(kind):
    """A decode step of a layer with a query norm weight and fp8 outputs (128-channel blocks):
    C4 (indexer, top-k, sparse attention; 3 sequences at ~9K context, one completing a block)
    and C128 (dense; 8 sequences at 65K context)."""
    if kind == "c4":
        spec = dataclasses.replace(W.C4_SPEC, q_norm=True, out_dtype="fp8")
        la = W.make_layer(spec, 3, 9000 // 4 + 4, seed=81, outlier_frac=0.05)
        st = W.make_step(spec, 3, [9003, 9000, 9130], seed=82, q_std=2.0)
    else:
        spec = dataclasses.replace(W.C128_SPEC, q_norm=True, out_dtype="fp8")
        la = W.make_layer(spec, 8, 65536 // 128, seed=83, value_std=1 / np.sqrt(512))
        st = W.make_step(spec, 8, 65536, seed=84, q_std=1.0)
    dl = dsv4.DeviceLayer.from_arrays(la)
    ol = OA.layer_state(la)
    _step_and_check(dl, ol, spec, st)


def test_c4_fp4_indexer_cache_steps():
    """The C4 step with an fp4 (e2m1) indexer cache: 6 sequences at 9K-40K context, two
    consecutive steps; at the second, sequences 0..2 complete a block and their new indexer
    entry (encoded to e2m1 by the step's own prologue, scored by the top-k kernel from the
    packed codes) is built to rank among their top k. Queries are drawn as in the benchmark
    workload (std 1), the scale the output bound assumes."""
    spec = W.C4_FP4_SPEC
    B = 6
    pos0 = np.array([9002, 12006, 40002, 9000, 17001, 33333], np.int64)
    la = W.make_layer(spec, B, int(pos0.max()) // 4 + 8, seed=91, outlier_frac=0.05)
    dl = dsv4.DeviceLayer.from_arrays(la)
    ol = OA.layer_state(la)
    for i in range(2):
        st = W.make_step(spec, B, (pos0 + i).tolist(), seed=92 + i)
        must = {s: _rank_new_index_entry(spec, st, s, ol) for s in range(3)} if i == 1 else None
        _step_and_check(dl, ol, spec, st, must_select=must)
