"""The benchmark's host helpers that need no GPU."""

import torch

import bench
import compressed_sparse_kv_dsv4_b200 as dsv4
import synthetic as W


def test_packed_step_inputs_are_views_of_one_buffer_with_the_same_bytes():
    la, sets = W.c4_sparse(seed=3, B=3, context=2048, steps=1)
    ds = dsv4.DeviceStep.from_arrays(la.spec, sets[0], "cpu")
    host, dev, packed = bench.pack_step_inputs(ds, torch.device("cpu"))
    assert host.numel() == dev.numel() and torch.equal(host, dev)
    lo, hi = dev.data_ptr(), dev.data_ptr() + dev.numel()
    raw = 0
    for n in bench.STEP_INPUTS:
        a, b = getattr(ds, n), getattr(packed, n)
        assert a.dtype == b.dtype and a.shape == b.shape, n
        assert torch.equal(a.reshape(-1).view(torch.uint8), b.reshape(-1).view(torch.uint8)), n
        assert lo <= b.data_ptr() and b.data_ptr() + b.numel() * b.element_size() <= hi, n
        assert (b.data_ptr() - lo) % 256 == 0, n
        raw += a.numel() * a.element_size()
    # the copy carries the step's bytes plus at most 255 bytes of alignment per tensor
    assert raw <= host.numel() <= raw + 255 * len(bench.STEP_INPUTS)
    # the rest of the step (outputs, positions, status) is the same
    assert packed.out is ds.out and packed.pos is ds.pos and packed.d_status is ds.d_status
