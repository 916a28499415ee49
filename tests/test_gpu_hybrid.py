"""GPU parity of dsv4_hybrid_decode on the benchmark workloads, against the oracle.

  tiny C4, fp32     built end to end from hidden states (prefill through the GPU's own
                    compressor and window insert on one side, the oracle's on the other),
                    then one decode step at position 4096.
  C128 dense, bf16  B = 8, 65536-token context.
  C4 sparse, fp8    B = 32, 131072-token context (the benchmark's launch configuration).
  1M stack          two C4 + two C128 layers, B = 4, 16 consecutive decode steps; the oracle
                    follows every state update and checks the attention at steps 0, 3 and 15.
"""

import numpy as np
import pytest
import torch

import compressed_sparse_kv_dsv4_b200 as dsv4
import oracle.dsv4_oracle as O
import synthetic as W
from oracle import adapters as OA
from tests.parity import check_output, check_topk, decode_out, input_class, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _new_entry_set(spec, pos):
    """Entries the decode step itself appends (built by each side's own compressor)."""
    n_before = pos // spec.m
    return set(range(n_before, (pos + 1) // spec.m))


def _step_and_check(dl, ol, spec, st, seqs=None, attend=True, extra_entries=None):
    ds = dsv4.DeviceStep.from_arrays(spec, st)
    dsv4.hybrid_decode(dl, ds)
    torch.cuda.synchronize()
    assert ds.d_status.item() == 0, f"device status {ds.d_status.item()}"
    oin = OA.step_inputs(spec, st)
    O.decode_update(ol, oin)
    if not attend:
        return None
    res = O.decode_attend(ol, oin, seqs)
    out = decode_out(ds.out)
    idx = ds.topk_idx.cpu().numpy() if ds.topk_idx is not None else None
    swaps = 0
    for s, (o, sel, scores) in res.items():
        if spec.kind == "c4":
            n_c = O.visible_entries(int(st.pos[s]), spec.m)
            swaps += check_topk(idx[s], scores, spec.k, n_c, f"seq {s}", allow_extra=extra_entries)
        check_output(out[s], o, input_class(spec), f"seq {s}", stored_bf16=spec.out_dtype == "bf16")
    return swaps


def _compare_caches(dl, ol, spec, s_range, entries, ctx):
    pages = dsv4.to_numpy_codes(dl.cache.pages, spec.cache_dtype)
    for s in s_range:
        for j in entries:
            pg, sl = ol.main_cache.locate(s, j)
            g = O.decode_rows(pages[pg, sl], dl.cache.scales[pg, sl].item(), spec.cache_dtype)
            r = ol.main_cache.read(s, j)
            tol = 2e-5 if spec.cache_dtype == "f32" else (2 ** -7 if spec.cache_dtype == "bf16" else 2 ** -3)
            assert np.all(np.abs(g - r) <= tol * np.abs(r).max() + 1e-7), f"{ctx}: entry {j} of seq {s}"


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
    _compare_caches(dl, ol, spec, [0], range(L // spec.m), "prefix")
    swaps = _step_and_check(dl, ol, spec, wl.step)
    assert swaps <= 2


def test_c128_dense_bf16_full_size():
    la, steps = W.c128_dense_bf16()
    spec = la.spec
    dl = dsv4.DeviceLayer.from_arrays(la)
    ol = OA.layer_state(la)
    _step_and_check(dl, ol, spec, steps[0])


@pytest.mark.slow
def test_c4_sparse_131k_full_size():
    la, steps = W.c4_sparse(steps=5)
    spec = la.spec
    dl = dsv4.DeviceLayer.from_arrays(la)
    ol = OA.layer_state(la)
    # five consecutive steps: positions 131072..131076; the block of 131072..131075 completes at step 3
    for i, st in enumerate(steps):
        attend = i in (0, 3, 4)
        _step_and_check(dl, ol, spec, st, seqs=range(la.B) if attend else None, attend=attend,
                        extra_entries=set(range(32768, 32770)))
    # the entry completed at step 3 (index 32768) was built by each side's compressor
    _compare_caches(dl, ol, spec, range(la.B), [32768], "appended entry")


@pytest.mark.slow
def test_stack_1m_sixteen_steps():
    layers, step_sets = W.stack_1m(steps=16)
    dls = [dsv4.DeviceLayer.from_arrays(la) for la in layers]
    ols = [OA.layer_state(la) for la in layers]
    for i in range(16):
        for li, la in enumerate(layers):
            spec = la.spec
            attend = i in (0, 3, 15)
            n0 = (1 << 20) // spec.m
            _step_and_check(dls[li], ols[li], spec, step_sets[li][i], attend=attend,
                            extra_entries=set(range(n0, n0 + 8)))
    for li, la in enumerate(layers):
        if la.spec.kind == "c4":
            n0 = (1 << 20) // 4
            _compare_caches(dls[li], ols[li], la.spec, range(la.B), range(n0, n0 + 4), f"layer {li}")
