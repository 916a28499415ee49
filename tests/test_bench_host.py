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


def test_algorithmic_byte_counts():
    """The byte counts behind the bench's fractions, against the per-sequence figures worked
    out by hand: C3 (32768 fp8 indexer keys of 128 B + a 4 B scale; 640 attended rows of
    512 B + 4 B; bf16 query and output; the step's updates), its fp4 variant (64 B keys), the
    dense C128 step and the compressor prefill."""
    import bench

    b = bench.algorithmic_bytes_per_seq(32768)
    assert b["indexer"] == 32768 * 132 + 64 * 128 + 64 * 4 + 64 * 2 == 4_333_952
    assert b["attention"] == 640 * 516 + 64 * 512 * 2 * 2 == 461_312
    assert b["total"] == 4_803_460
    assert bench.c4_step_bytes_per_seq(32768) * 32 == 153_710_720
    f4 = bench.algorithmic_bytes_per_seq(32768, idx_row_bytes=64)
    assert f4["indexer"] == 32768 * 68 + 64 * 128 + 64 * 4 + 64 * 2
    assert f4["total"] - b["total"] == f4["indexer"] - b["indexer"]
    # dense C128: every entry and the window rows in bf16, q and o, the updates
    assert bench.c128_bytes_per_seq(512) == (512 + 128) * 1024 + 2 * 64 * 512 * 2 + (2 * 512 * 2 + 2 * 512 * 4 + 1024)
    # compressor prefill: 8 x 4096 bf16 tokens (kv + gate), 1024 entries per sequence at m = 4
    assert bench.prefill_bytes(32768, 8, 4) == 32768 * 2048 + 8 * 1024 * 1024 + 8 * 4 * 4096


def test_step_flop_counts():
    """The C3 step's tensor-core FLOPs: 17.2 GFLOP of indexer products and 2.7 GFLOP of attention
    for 32 sequences."""
    import bench

    f = bench.c4_step_flops_per_seq(32768)
    assert f["indexer"] * 32 == 2 * 64 * 128 * 32768 * 32 == 17_179_869_184
    assert f["attention"] * 32 == 4 * 64 * 640 * 512 * 32 == 2_684_354_560
