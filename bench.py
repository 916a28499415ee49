#!/usr/bin/env python
"""Decode-step benchmark of the hybrid-attention library on B200.

Workload (per GPU): one C4 layer decode step for B = 32 sequences at a 131072-token context
(32768 fp8 C4 entries per sequence, top-512 of a 64-head x 128-dim fp8 lightning indexer,
a 128-token fp8 sliding window, 64 query heads, KV dim 512, bf16 queries and outputs), on
seeded synthetic inputs. Each step appends one token per sequence; positions cycle over
131072..131583 so the context stays at 131K.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) every rank runs its own 32 sequences (weak scaling, no
data-path collective); the step time is the max over ranks. Rank 0 prints one JSON line.
"""

from __future__ import annotations

import argparse
import ctypes as C
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

B_PER_GPU = 32
CONTEXT = 131072
POS_CYCLE = 512
N_INPUT_SETS = 8
FLUSH_BYTES = 256 << 20
METRIC = "hybrid-attn decode tokens/s (C4 layer, 131072-token context, top-512 + SWA-128)"
UNIT = "tokens/s"

SPEC_ROWS = dict(D=512, H=64, k=512, W=128, H_I=64, d_I=128)


def algorithmic_bytes_per_seq(n_c: int, out_bytes: int = 2, idx_row_bytes: int = SPEC_ROWS["d_I"]) -> dict:
    """Bytes one sequence's decode step must move (fp8 caches with a 4-byte row scale).

    indexer: every visible indexer key row (128 B + scale); attention: the k selected
    rows and the W window rows (512 B + scale), the bf16 query and the output (out_bytes
    per value); updates:
    the new token's kv/gate and indexer kv/gate (bf16) read, the two compressor ring
    slots (float32) and the window row written; the indexer query, its scales and weights.
    """
    D, H, k, W, H_I, d_I = (SPEC_ROWS[x] for x in ("D", "H", "k", "W", "H_I", "d_I"))
    idx = n_c * (idx_row_bytes + 4)  # idx_row_bytes: d_I for fp8 keys, d_I / 2 for fp4
    attn = (k + W) * (D + 4) + H * D * 2 + H * D * out_bytes
    upd = 2 * D * 2 + 2 * d_I * 2 + 2 * D * 4 + 2 * d_I * 4 + (D + 4)  # appended cache rows: under 1/m per step
    qidx = H_I * d_I + H_I * 4 + H_I * 2
    return dict(indexer=idx + qidx, attention=attn, updates=upd, total=idx + qidx + attn + upd)


def c128_bytes_per_seq(n_c: int, D: int = 512, H: int = 64, W: int = 128) -> int:
    """Bytes one sequence's dense C128 layer step must move (bf16 caches): every visible entry
    and the W window rows (2D bytes each), the bf16 query and output, and the updates (the new
    token's kv and gate read, the state slot (float32 kv + gate) and the window row written)."""
    return (n_c + W) * 2 * D + 2 * H * D * 2 + (2 * D * 2 + 2 * D * 4 + 2 * D)


def c4_step_flops_per_seq(n_c: int) -> dict:
    """Tensor-core FLOPs of one sequence's C4 step: the indexer's q . k for every visible entry
    (2 H_I d_I each) and the attention's two products over the k + W keys (4 H D each)."""
    D, H, k, W, H_I, d_I = (SPEC_ROWS[x] for x in ("D", "H", "k", "W", "H_I", "d_I"))
    idx = 2 * H_I * d_I * n_c
    attn = 4 * H * (k + W) * D
    return dict(indexer=idx, attention=attn, total=idx + attn)


def c4_step_bytes_per_seq(n_c: int) -> int:
    return algorithmic_bytes_per_seq(n_c)["total"]


def prefill_bytes(T: int, B: int, m: int, D: int = 512, cache_bytes_per_row: int = 1024) -> int:
    """Bytes one compressor must move for a prefill of T bf16 tokens over B sequences of T/B
    tokens each (starting at position 0): the kv and gate rows read (2D bf16 each), one
    cache row per completed block written, and the ring state of each sequence's last m
    tokens written (float32 kv + gate)."""
    per = T // B
    return T * 2 * D * 2 + B * (per // m) * cache_bytes_per_row + B * min(m, per) * 2 * D * 4


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None

    def __enter__(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                                          "-lms", "100", "-i", self.gpu_id], stdout=subprocess.PIPE,
                                         stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 9:
                self.rows.append(parts)

    def summary(self, t_start: float, t_end: float) -> dict:
        rows = getattr(self, "rows", [])
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[5:9]) if v.lower() == "active"})
        load = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": float(np.median(load)) if load else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- distributed
def dist_setup(n_gpus: int, backend: str | None = None):
    """Rank, world size and local rank from the torchrun environment; joins the process
    group when world > 1 (nccl on GPUs; gloo where there is no GPU, as in the CPU tests)."""
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = backend or ("nccl" if torch.cuda.is_available() else "gloo")
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest x over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(rank: int) -> int:
    """Seed of a rank's own sequences: ranks decode disjoint, independent batches."""
    return 2 + 1000 * rank


def job_tokens_per_s(world: int, ms_max: float) -> float:
    """Whole-job decode tokens/s: every rank's sequences over the slowest rank's step."""
    return world * B_PER_GPU / (ms_max * 1e-3)


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(la, steps, budget_s: float, min_seqs: int = 2):
    """Time the oracle's decode step on whole sequences until budget_s is spent."""
    import oracle.dsv4_oracle as O
    from oracle import adapters as OA

    spec = la.spec
    ol = OA.layer_state(la)
    oin = OA.step_inputs(spec, steps[0])
    done, t0 = 0, time.perf_counter()
    O.decode_update(ol, oin)  # the update part of every sequence (cheap)
    for s in range(la.B):
        O.decode_attend(ol, oin, [s])
        done += 1
        if done >= min_seqs and time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return done, dt


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info

        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return 1


def kernel_sources_sha256() -> str:
    """Hash of the sources the indexer kernel is compiled from."""
    import hashlib

    h = hashlib.sha256()
    for f in ("indexer.cu", "common.cuh", "internal.h"):
        with open(os.path.join(ROOT, "compressed_sparse_kv_dsv4_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def indexer_traffic():
    """DRAM bytes (read + write) per indexer launch at this workload, from the committed ncu
    summary; None when there is none or the kernel's sources changed since it was taken."""
    try:
        rec = json.load(open(os.path.join(ROOT, "profiles", "indexer_traffic.json")))
    except (OSError, ValueError):
        return None
    if rec.get("sources_sha256") != kernel_sources_sha256():
        return None
    return rec.get("dram_bytes_per_launch")


STEP_INPUTS = ("kv", "gate", "idx_kv", "idx_gate", "q", "q_idx", "q_idx_scale", "w")


def pack_step_inputs(ds, dev):
    """A copy of step ds whose input tensors are views into one device buffer (each at a
    256-byte offset), with a pinned host mirror of that buffer: (host, device, step)."""
    import dataclasses

    import torch

    offs, size = [], 0
    for n in STEP_INPUTS:
        t = getattr(ds, n)
        offs.append(size)
        size += (t.numel() * t.element_size() + 255) // 256 * 256
    dbuf = torch.zeros(size, dtype=torch.uint8, device=dev)
    views = {}
    for n, off in zip(STEP_INPUTS, offs):
        t = getattr(ds, n)
        v = dbuf[off:off + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
        v.copy_(t)
        views[n] = v
    return dbuf.cpu().pin_memory() if dbuf.is_cuda else dbuf.clone(), dbuf, dataclasses.replace(ds, **views)


# ----------------------------------------------------------------------------- extra legs
def event_mean_ms(stream, fn, iters: int, flush, warm: int = 3) -> float:
    """Mean duration of fn() over `iters` runs, CUDA events on `stream`, L2 flushed before each."""
    import torch

    for j in range(warm):
        flush.fill_(j & 0xFF)
        fn(j)
    torch.cuda.synchronize()
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(iters)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(iters)]
    for j in range(iters):
        flush.fill_(j & 0xFF)
        e0[j].record(stream)
        fn(warm + j)
        e1[j].record(stream)
    torch.cuda.synchronize()
    return float(np.mean([e0[j].elapsed_time(e1[j]) for j in range(iters)]))


def leg_compress_prefill(lib, dev, stream, flush, hbm_peak: float, iters: int = 20) -> dict:
    """The compressor prefill workload: 8 x 4096 bf16 tokens (D = 512) into a C4 and a C128
    compressor (pool + RMSNorm + RoPE + bf16 insert + ring state), each dsv4_compress call
    timed alone and both together."""
    import torch

    import compressed_sparse_kv_dsv4_b200 as dsv4
    from compressed_sparse_kv_dsv4_b200 import _abi as A
    import synthetic as W

    wl = W.compressor_prefill()
    B, T = wl.start_pos.shape[0], int(wl.cu_seqlens[-1])
    cu = torch.from_numpy(wl.cu_seqlens).to(dev)
    sp = torch.from_numpy(wl.start_pos).to(dev)
    calls = []
    for la, kv, gate in ((wl.layer4, wl.kv4, wl.gate4), (wl.layer128, wl.kv128, wl.gate128)):
        spec = la.spec
        dl = dsv4.DeviceLayer.from_arrays(la, dev)
        kvd, gd = dsv4.to_device_codes(kv, "bf16", dev), dsv4.to_device_codes(gate, "bf16", dev)
        a = A.CompressArgs(batch=B, total_tokens=T, kv=kvd.data_ptr(), gate=gd.data_ptr(), kv_dtype=A.BF16,
                           cu_seqlens=cu.data_ptr(), start_pos=sp.data_ptr(), gamma=dl.gamma.data_ptr(), eps=spec.eps,
                           rope=A.Rope(spec.rope_dims, spec.rope_base), state=dl.state.struct(),
                           cache=dl.cache.struct(), d_status=None)
        calls.append((spec.m, a, (dl, kvd, gd)))
    sh = C.c_void_p(stream.cuda_stream)
    out = {"workload": "compressor_prefill_8x4096", "tokens": T, "kv_dim": 512, "cache": "bf16",
           "input": "bf16 kv + per-channel gate"}
    total_bytes, total_ms = 0, 0.0
    for m, a, _keep in calls:
        ms = event_mean_ms(stream, lambda j, a=a: A.check("dsv4_compress", lib.dsv4_compress(C.byref(a), sh)),
                           iters, flush)
        byts = prefill_bytes(T, B, m)
        out[f"c{m}"] = {"ms": round(ms, 5), "algorithmic_bytes": byts, "gbs": round(byts / ms / 1e6, 1),
                        "frac": round(byts / ms / 1e6 / hbm_peak, 4)}
        total_bytes += byts
        total_ms += ms
    both = event_mean_ms(stream, lambda j: [A.check("dsv4_compress", lib.dsv4_compress(C.byref(a), sh))
                                            for _m, a, _k in calls], iters, flush)
    out["both"] = {"ms": round(both, 5), "algorithmic_bytes": total_bytes, "gbs": round(total_bytes / both / 1e6, 1),
                   "frac": round(total_bytes / both / 1e6 / hbm_peak, 4), "tokens_per_s": round(T / (both * 1e-3), 1)}
    return out


def leg_compress_project(lib, dev, stream, flush, peaks: dict, iters: int = 10) -> dict:
    """The compressor prefill with its projection: 8 x 4096 tokens of bf16 hidden states
    (hidden 4096) projected on the tensor cores into kv and gate (D = 512) for a C4 and a C128
    compressor, each then compressed (dsv4_compress_project, one call per compressor).
    FLOPs counted: the projections only, 2 T hidden 2D per compressor."""
    import torch

    import compressed_sparse_kv_dsv4_b200 as dsv4
    from compressed_sparse_kv_dsv4_b200 import _abi as A
    import synthetic as W

    wl = W.projection_prefill()
    B, T = wl.start_pos.shape[0], int(wl.cu_seqlens[-1])
    Hd, D = wl.hidden.shape[1], wl.layer4.spec.D
    cu = torch.from_numpy(wl.cu_seqlens).to(dev)
    sp = torch.from_numpy(wl.start_pos).to(dev)
    hid = dsv4.to_device_codes(wl.hidden, "bf16", dev)
    calls = []
    for la, w in ((wl.layer4, wl.w4), (wl.layer128, wl.w128)):
        spec = la.spec
        dl = dsv4.DeviceLayer.from_arrays(la, dev)
        wd = dsv4.to_device_codes(w, "bf16", dev)
        c = A.CompressArgs(batch=B, total_tokens=T, kv=None, gate=None, kv_dtype=A.BF16, cu_seqlens=cu.data_ptr(),
                           start_pos=sp.data_ptr(), gamma=dl.gamma.data_ptr(), eps=spec.eps,
                           rope=A.Rope(spec.rope_dims, spec.rope_base), state=dl.state.struct(),
                           cache=dl.cache.struct(), d_status=None)
        a = A.CompressProjectArgs(c=c, hidden=hid.data_ptr(), w=wd.data_ptr(), hidden_dim=Hd)
        ws = torch.empty(lib.dsv4_compress_project_workspace_size(C.byref(a)), dtype=torch.uint8, device=dev)
        calls.append((spec.m, a, ws, (dl, wd)))
    sh = C.c_void_p(stream.cuda_stream)
    flops = 2.0 * T * Hd * 2 * D  # per compressor
    bf16_peak = float(peaks.get("bf16_tflops", 1590.0))
    out = {"workload": "compressor_prefill_projected_8x4096", "tokens": T, "hidden": Hd, "kv_dim": D,
           "cache": "bf16", "flops_per_compressor": flops, "peak_tflops": bf16_peak,
           "peak_source": "measured" if "bf16_tflops" in peaks else "fallback"}
    total = 0.0
    for m, a, ws, _keep in calls:
        ms = event_mean_ms(stream, lambda j, a=a, ws=ws: A.check("dsv4_compress_project", lib.dsv4_compress_project(
            C.byref(a), C.c_void_p(ws.data_ptr()), ws.numel(), sh)), iters, flush)
        tf = flops / (ms * 1e-3) / 1e12
        out[f"c{m}"] = {"ms": round(ms, 5), "tflops": round(tf, 1), "frac": round(tf / bf16_peak, 4)}
        total += ms
    out["both"] = {"ms": round(total, 5), "tflops": round(2 * flops / (total * 1e-3) / 1e12, 1),
                   "frac": round(2 * flops / (total * 1e-3) / 1e12 / bf16_peak, 4),
                   "tokens_per_s": round(T / (total * 1e-3), 1)}
    del calls, hid
    torch.cuda.empty_cache()
    return out


def leg_stack_1m(lib, dev, stream, flush, hbm_peak: float, steps: int = 16) -> dict:
    """The 1M-context mixed stack: two C4 layers (262144 fp8 entries, top-512) and two C128
    layers (8192 bf16 entries), 4 sequences; one step = the four layers' dsv4_hybrid_decode
    calls, each sequence appending one token per layer. `steps` consecutive steps after three
    warm-up steps, the L2 flushed before each."""
    import torch

    import compressed_sparse_kv_dsv4_b200 as dsv4
    from compressed_sparse_kv_dsv4_b200 import _abi as A
    import synthetic as W

    B, ctx = 4, 1 << 20
    layers, step_sets = W.stack_1m(B=B, context=ctx, steps=1)
    dls = [dsv4.DeviceLayer.from_arrays(la, dev) for la in layers]
    dss = [dsv4.DeviceStep.from_arrays(la.spec, ss[0], dev) for la, ss in zip(layers, step_sets)]
    total = steps + 3
    pos = torch.tensor([[ctx + i] * B for i in range(total)], dtype=torch.int32, device=dev)
    wss = [dl.workspace(B) for dl in dls]
    Ls = [dl.struct() for dl in dls]
    Ss = []
    for ds in dss:
        row = []
        for i in range(total):
            S = ds.struct()
            S.pos = pos[i].data_ptr()
            row.append(S)
        Ss.append(row)
    sh = C.c_void_p(stream.cuda_stream)

    def step(i):
        for li in range(4):
            A.check("dsv4_hybrid_decode", lib.dsv4_hybrid_decode(C.byref(Ls[li]), C.byref(Ss[li][i]),
                                                                  C.c_void_p(wss[li].data_ptr()), wss[li].numel(), sh))

    n0 = lib.dsv4_launch_count()
    ms = event_mean_ms(stream, step, steps, flush, warm=3)
    launches = (lib.dsv4_launch_count() - n0) // total
    status = [int(ds.d_status.item()) for ds in dss]
    byts = B * (2 * c4_step_bytes_per_seq(ctx // 4) + 2 * c128_bytes_per_seq(ctx // 128))
    res = {"workload": "stack_1m", "batch": B, "context": ctx, "layers": "C4, C128, C4, C128", "steps": steps,
           "ms_per_step": round(ms, 5), "tokens_per_s": round(B / (ms * 1e-3), 1), "algorithmic_bytes": byts,
           "gbs": round(byts / ms / 1e6, 1), "pct_of_8tbs": round(100 * byts / ms / 1e6 / 8000.0, 1),
           "frac": round(byts / ms / 1e6 / hbm_peak, 4), "launches_per_step": launches, "device_status": status,
           "l2": "flushed between steps (256 MiB write)"}
    del dls, dss, wss
    torch.cuda.empty_cache()
    return res


def leg_c4_fp4_indexer(lib, dev, stream, flush, hbm_peak: float, steps: int = 50) -> dict:
    """The benchmark's C4 step (32 sequences, 131072-token context) with an fp4 (e2m1)
    indexer-key cache: 64 bytes + a float32 scale per entry instead of 128 + 4. One step =
    one dsv4_hybrid_decode call; the scoring kernel is also timed alone."""
    import torch

    import compressed_sparse_kv_dsv4_b200 as dsv4
    from compressed_sparse_kv_dsv4_b200 import _abi as A
    from compressed_sparse_kv_dsv4_b200.binding import indexer_args
    import synthetic as W

    spec = W.C4_FP4_SPEC
    la, sets = W.c4_sparse(seed=7, B=B_PER_GPU, context=CONTEXT, steps=1, spec=spec)
    dl = dsv4.DeviceLayer.from_arrays(la, dev)
    ds = dsv4.DeviceStep.from_arrays(spec, sets[0], dev)
    total = steps + 3
    pos = torch.tensor([[CONTEXT + (i % POS_CYCLE)] * B_PER_GPU for i in range(total)], dtype=torch.int32,
                       device=dev)
    ws = dl.workspace(B_PER_GPU)
    L = dl.struct()
    Ss = []
    for i in range(total):
        S = ds.struct()
        S.pos = pos[i].data_ptr()
        Ss.append(S)
    sh = C.c_void_p(stream.cuda_stream)
    n0 = lib.dsv4_launch_count()
    ms = event_mean_ms(stream, lambda i: A.check("dsv4_hybrid_decode", lib.dsv4_hybrid_decode(
        C.byref(L), C.byref(Ss[i]), C.c_void_p(ws.data_ptr()), ws.numel(), sh)), steps, flush, warm=3)
    launches = (lib.dsv4_launch_count() - n0) // total
    status = int(ds.d_status.item())
    n_c = CONTEXT // spec.m
    n_ent = torch.full((B_PER_GPU,), n_c, dtype=torch.int32, device=dev)
    ia = indexer_args(ds.q_idx, ds.w, dl.idx_cache, n_ent, spec.k, q_dtype="fp8", w_dtype="bf16",
                      q_scale=ds.q_idx_scale, d_status=ds.d_status)
    sc_ld = (dl.idx_cache.block_table.shape[1] * (A.PAGE_POSITIONS // spec.m) + 3) // 4 * 4
    sc_buf = torch.empty((B_PER_GPU, sc_ld), dtype=torch.float32, device=dev)
    sc_ms = event_mean_ms(stream, lambda j: A.check("dsv4_indexer_scores", lib.dsv4_indexer_scores(
        C.byref(ia), C.c_void_p(sc_buf.data_ptr()), sc_ld, sh)), steps, flush)
    byts = algorithmic_bytes_per_seq(n_c, out_bytes=2, idx_row_bytes=spec.d_I // 2)
    step_b, ix_b = byts["total"] * B_PER_GPU, byts["indexer"] * B_PER_GPU
    res = {"workload": "c4_sparse_131k_fp4_indexer", "batch": B_PER_GPU, "context": CONTEXT,
           "indexer_cache": "e2m1, 64 B + fp32 scale per entry", "ms_per_step": round(ms, 5),
           "tokens_per_s": round(B_PER_GPU / (ms * 1e-3), 1), "step_algorithmic_bytes": step_b,
           "step_frac": round(step_b / ms / 1e6 / hbm_peak, 4),
           "indexer_scores_ms": round(sc_ms, 5), "indexer_algorithmic_bytes": ix_b,
           "indexer_gbs": round(ix_b / sc_ms / 1e6, 1), "indexer_frac": round(ix_b / sc_ms / 1e6 / hbm_peak, 4),
           "launches_per_step": launches, "device_status": status, "l2": "flushed between steps (256 MiB write)"}
    del dl, ds, ws, sc_buf
    torch.cuda.empty_cache()
    return res


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args):
    import torch

    import compressed_sparse_kv_dsv4_b200 as dsv4
    from compressed_sparse_kv_dsv4_b200 import _abi as A
    import synthetic as W

    rank, world, local = dist_setup(args.gpus)
    dev = torch.device("cuda", local)
    lib = dsv4.load()
    la, sets = W.c4_sparse(seed=shard_seed(rank), B=B_PER_GPU, context=CONTEXT, steps=N_INPUT_SETS)
    spec = la.spec
    dl = dsv4.DeviceLayer.from_arrays(la, dev)
    dsteps = [dsv4.DeviceStep.from_arrays(spec, st, dev) for st in sets]
    total = args.warmup + args.steps
    pos_table = torch.tensor([[CONTEXT + (i % POS_CYCLE)] * B_PER_GPU for i in range(total)],
                             dtype=torch.int32, device=dev)
    ws = dl.workspace(B_PER_GPU)
    L = dl.struct()
    stream = torch.cuda.current_stream(dev)
    sh = C.c_void_p(stream.cuda_stream)
    structs = []
    for i in range(total):
        ds = dsteps[i % N_INPUT_SETS]
        S = ds.struct()
        S.pos = pos_table[i].data_ptr()
        structs.append(S)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(i):
        A.check("dsv4_hybrid_decode", lib.dsv4_hybrid_decode(C.byref(L), C.byref(structs[i]),
                                                              C.c_void_p(ws.data_ptr()), ws.numel(), sh))

    for i in range(args.warmup):
        flush.fill_(i & 0xFF)
        step(i)
    torch.cuda.synchronize()
    ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    gpu_id = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    with ClockSampler(gpu_id) as clk:
        barrier(world)
        torch.cuda.synchronize()
        t_a = time.time()
        launches0 = lib.dsv4_launch_count()
        for j in range(args.steps):
            flush.fill_(j & 0xFF)
            ev0[j].record(stream)
            step(args.warmup + j)
            ev1[j].record(stream)
        launches = lib.dsv4_launch_count() - launches0
        torch.cuda.synchronize()
        barrier(world)
        t_b = time.time()
    times = np.array([ev0[j].elapsed_time(ev1[j]) for j in range(args.steps)])
    ms_local = float(times.mean())
    ms = max_over_ranks(ms_local, world)
    status = int(dsteps[0].d_status.item())

    # ---- dominant kernel alone: the lightning indexer + top-k, same launch configuration
    st0 = dsteps[0]
    n_c = CONTEXT // spec.m
    n_ent = torch.full((B_PER_GPU,), n_c, dtype=torch.int32, device=dev)
    idx_out = torch.empty((B_PER_GPU, spec.k), dtype=torch.int32, device=dev)
    from compressed_sparse_kv_dsv4_b200.binding import indexer_args
    ia = indexer_args(st0.q_idx, st0.w, dl.idx_cache, n_ent, spec.k, q_dtype="fp8", w_dtype="bf16",
                      q_scale=st0.q_idx_scale, idx=idx_out, d_status=st0.d_status)
    iws = torch.empty(lib.dsv4_indexer_workspace_size(C.byref(ia)), dtype=torch.uint8, device=dev)
    k_iters = min(args.steps, 200)
    e0 = [torch.cuda.Event(enable_timing=True) for _ in range(k_iters)]
    e1 = [torch.cuda.Event(enable_timing=True) for _ in range(k_iters)]
    for j in range(3):
        lib.dsv4_indexer_topk(C.byref(ia), C.c_void_p(iws.data_ptr()), iws.numel(), sh)
    for j in range(k_iters):
        flush.fill_(j & 0xFF)
        e0[j].record(stream)
        A.check("dsv4_indexer_topk", lib.dsv4_indexer_topk(C.byref(ia), C.c_void_p(iws.data_ptr()), iws.numel(), sh))
        e1[j].record(stream)
    torch.cuda.synchronize()
    ix_ms = float(np.mean([e0[j].elapsed_time(e1[j]) for j in range(k_iters)]))
    # the scoring kernel alone (dsv4_indexer_scores: the same launch without the selection)
    sc_ld = (dl.idx_cache.block_table.shape[1] * (A.PAGE_POSITIONS // spec.m) + 3) // 4 * 4
    sc_buf = torch.empty((B_PER_GPU, sc_ld), dtype=torch.float32, device=dev)
    sc_ms = event_mean_ms(stream, lambda j: A.check("dsv4_indexer_scores", lib.dsv4_indexer_scores(
        C.byref(ia), C.c_void_p(sc_buf.data_ptr()), sc_ld, sh)), k_iters, flush)

    # ---- end to end through the public API: inputs from pinned host memory, output back,
    # pipelined as a serving loop runs it: step j's inputs cross on a copy stream while step
    # j - 1 computes, and its output returns on a second copy stream while step j + 1
    # computes. A step's eight input tensors live in one device buffer (views at 256-byte
    # offsets) with a pinned host mirror of the same layout, so they cross in one copy; the
    # positions in a second one. Each of the 8 input sets has its own buffers; a set is
    # refilled only after the step that last used it computed and its output was read back.
    # No L2 flush here: a step reads 154 MB, more than the 126 MB L2.
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    pos_host = pos_table.cpu().pin_memory()
    packed = [pack_step_inputs(ds, dev) for ds in dsteps]  # (host mirror, device buffer, step)
    pos_devs = [torch.empty(B_PER_GPU, dtype=torch.int32, device=dev) for _ in packed]
    e2e_structs = []
    for (hbuf, dbuf, ds_e), pdv in zip(packed, pos_devs):
        S = ds_e.struct()
        S.pos = pdv.data_ptr()
        e2e_structs.append(S)
    out_hosts = [torch.empty(dsteps[0].out.shape, dtype=dsteps[0].out.dtype).pin_memory() for _ in range(2)]
    h2d = packed[0][0].numel() + B_PER_GPU * 4
    d2h = out_hosts[0].numel() * out_hosts[0].element_size()
    e2e_steps = min(args.steps, 200)
    ev_in = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_cmp = [torch.cuda.Event() for _ in range(e2e_steps)]
    ev_out = [torch.cuda.Event() for _ in range(e2e_steps)]
    t_first = torch.cuda.Event(enable_timing=True)
    t_last = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    t_first.record(s_in)
    for j in range(e2e_steps):
        i = args.warmup + j
        k = i % N_INPUT_SETS
        hbuf, dbuf, ds_e = packed[k]
        with torch.cuda.stream(s_in):
            if j >= N_INPUT_SETS:
                s_in.wait_event(ev_cmp[j - N_INPUT_SETS])
            dbuf.copy_(hbuf, non_blocking=True)
            pos_devs[k].copy_(pos_host[i], non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if j >= N_INPUT_SETS:
            stream.wait_event(ev_out[j - N_INPUT_SETS])
        A.check("dsv4_hybrid_decode", lib.dsv4_hybrid_decode(C.byref(L), C.byref(e2e_structs[k]),
                                                              C.c_void_p(ws.data_ptr()), ws.numel(), sh))
        ev_cmp[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[j])
            out_hosts[j % 2].copy_(ds_e.out, non_blocking=True)
            ev_out[j].record(s_out)
    t_last.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(t_first.elapsed_time(t_last) / e2e_steps, world)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()
        return

    byts = algorithmic_bytes_per_seq(n_c, out_bytes=4 if spec.out_dtype == "f32" else 2)
    step_bytes = byts["total"] * B_PER_GPU
    fl = c4_step_flops_per_seq(n_c)
    step_flops, ix_flops = fl["total"] * B_PER_GPU, fl["indexer"] * B_PER_GPU
    ix_bytes = byts["indexer"] * B_PER_GPU
    peaks = {}
    try:
        peaks = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        hbm_peak, peak_src = float(peaks["hbm_gbs"]), "measured"
    except Exception:  # noqa: BLE001
        hbm_peak, peak_src = 6650.0, "fallback"
    ix_gbs = ix_bytes / (ix_ms * 1e-3) / 1e9
    sc_gbs = ix_bytes / (sc_ms * 1e-3) / 1e9
    step_gbs = step_bytes / (ms * 1e-3) / 1e9
    traffic = indexer_traffic()
    value = job_tokens_per_s(world, ms)
    line = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp8", "data": "synthetic",
        "config": {"workload": "c4_sparse_131k", "batch_per_gpu": B_PER_GPU, "global_batch": world * B_PER_GPU,
                   "context": CONTEXT, "c4_entries": n_c, "topk": spec.k, "window": spec.W, "heads": spec.H,
                   "kv_dim": spec.D, "indexer": f"{spec.H_I} heads x {spec.d_I} fp8", "cache": "fp8 e4m3 + fp32 row scale",
                   "query": "bf16", "output": spec.out_dtype,
                   "arithmetic": "e4m3 x e4m3 indexer MMA, fp16-operand attention MMAs over e4m3 rows, f32 accumulate",
                   "parallelism": f"dp{world} (independent sequences)", "l2": "flushed between steps (256 MiB write)",
                   "positions": f"advance by one per step, cycling over {CONTEXT}..{CONTEXT + POS_CYCLE - 1}"},
        "hbm": {"step_algorithmic_bytes": step_bytes, "achieved_gbs": round(step_gbs, 1),
                "pct_of_8tbs": round(100 * step_gbs / 8000.0, 1),
                "pct_of_measured_copy": round(100 * step_gbs / hbm_peak, 1)},
        "tflops": {"step": round(step_flops / (ms * 1e-3) / 1e12, 1),
                   "indexer_alone": round(ix_flops / (sc_ms * 1e-3) / 1e12, 1),
                   "step_flops": step_flops, "note": "fp8 indexer and fp16 attention MMAs; HBM-bound"},
        "roofline": {"kernel": "indexer_tc_kernel (dsv4_indexer_scores)", "bound": "hbm",
                     "achieved": round(sc_gbs, 1), "peak": hbm_peak, "peak_source": peak_src, "unit": "GB/s",
                     "frac": round(sc_gbs / hbm_peak, 4), "traffic": traffic, "algorithmic_bytes_per_launch": ix_bytes,
                     "launch_ms": round(sc_ms, 5),
                     "call": {"name": "dsv4_indexer_topk: indexer_tc_kernel + topk_scores_kernel",
                              "launch_ms": round(ix_ms, 5), "achieved": round(ix_gbs, 1),
                              "frac": round(ix_gbs / hbm_peak, 4)}},
        "e2e": {"value": round(job_tokens_per_s(world, e2e_ms), 1), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5), "steps": e2e_steps,
                "timing": "from the first input copy to the last output copy, divided by the steps",
                "pipeline": "inputs and outputs on two copy streams overlap the neighbouring steps' kernels",
                "l2": "not flushed (a step reads 154 MB, more than the 126 MB L2)"},
        "gpu_launches": int(launches),
        "clocks": clk.summary(t_a, t_b),
        "device_status": status,
    }
    if world == 1 and not args.no_extra:
        line["compress_prefill"] = leg_compress_prefill(lib, dev, stream, flush, hbm_peak)
        line["c4_fp4_indexer"] = leg_c4_fp4_indexer(lib, dev, stream, flush, hbm_peak)
        line["compress_project"] = leg_compress_project(lib, dev, stream, flush, peaks)
        if not args.skip_1m:
            line["stack_1m"] = leg_stack_1m(lib, dev, stream, flush, hbm_peak)
    if world == 1 and not args.no_cpu_baseline:
        seqs, dt = oracle_sample(la, sets, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": round(seqs / dt, 3), "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "host_cores": os.cpu_count(),
                                "sample": f"{seqs} of {B_PER_GPU} sequences of one decode step (float64 oracle)"}
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


# ----------------------------------------------------------------------------- reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import synthetic as W

    la, sets = W.c4_sparse(seed=2, B=B_PER_GPU, context=CONTEXT, steps=1)
    per_step = []
    budget = max(1.0, 120.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        seqs, dt = oracle_sample(la, sets, budget_s=budget, min_seqs=1)
        if i >= args.warmup:
            per_step.append(seqs / dt)
    value = float(np.mean(per_step))
    cores = blas_threads()
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * B_PER_GPU / value, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "c4_sparse_131k", "batch_per_gpu": B_PER_GPU, "context": CONTEXT},
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": "each step: whole sequences of one C4 decode step until its time budget"},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the compressor-prefill and 1M-stack legs")
    ap.add_argument("--skip-1m", action="store_true", help="skip the 1M-stack leg")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
