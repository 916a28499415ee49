"""Thin Python binding of libdsv4.so: torch tensors in, ctypes structs out.

Every step of the decode path runs in the library's CUDA kernels; this module only
builds the argument structs from torch CUDA tensors and passes the caller's current
stream. It has no CPU fallback: without the built library every call raises.
"""

from __future__ import annotations

import ctypes as C
from dataclasses import dataclass, field

import numpy as np
import torch

from . import _abi as A

DT = {"f32": A.F32, "bf16": A.BF16, "fp8": A.FP8, "fp4": A.FP4}
TORCH_CODE_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16, "fp8": torch.uint8, "fp4": torch.uint8}


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return t.data_ptr()


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def to_device_codes(a: np.ndarray, dtype: str, device) -> torch.Tensor:
    """numpy codes (float32 / uint16 bf16 bits / uint8 e4m3) -> CUDA tensor of the code dtype."""
    a = np.ascontiguousarray(a)
    if dtype == "bf16":
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
    elif dtype in ("fp8", "fp4"):  # e4m3 codes, or e2m1 codes packed two per byte
        t = torch.from_numpy(a.view(np.uint8))
    else:
        t = torch.from_numpy(a.astype(np.float32, copy=False))
    return t.to(device, non_blocking=False)


def to_numpy_codes(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16)
    if dtype in ("fp8", "fp4"):
        return t.view(torch.uint8).numpy()
    return t.float().numpy()


@dataclass
class DeviceCache:
    pages: torch.Tensor        # [num_pages, 256/m, dim] codes
    scales: torch.Tensor       # [num_pages, 256/m] float32
    block_table: torch.Tensor  # [B, max_blocks] int32
    m: int
    dtype: str

    @property
    def dim(self) -> int:
        return self.pages.shape[2] * (2 if self.dtype == "fp4" else 1)  # fp4 rows: dim/2 bytes

    def struct(self) -> A.PagedCache:
        return A.PagedCache(_ptr(self.pages), _ptr(self.scales), _ptr(self.block_table), self.pages.shape[0],
                            self.block_table.shape[1], self.dim, self.m, DT[self.dtype])


@dataclass
class DeviceRing:
    rows: torch.Tensor    # [B, W, dim] codes
    scales: torch.Tensor  # [B, W] float32
    dtype: str

    def struct(self) -> A.WindowRing:
        return A.WindowRing(_ptr(self.rows), _ptr(self.scales), self.rows.shape[1], self.rows.shape[2], DT[self.dtype])


@dataclass
class DeviceState:
    buf: torch.Tensor  # [B, m, dim + gate_dim] float32
    dim: int

    def struct(self) -> A.CompressorState:
        return A.CompressorState(_ptr(self.buf), self.buf.shape[1], self.dim, self.buf.shape[2] - self.dim)


@dataclass
class DeviceLayer:
    kind: str
    H: int
    D: int
    gamma: torch.Tensor
    state: DeviceState
    cache: DeviceCache
    ring: DeviceRing
    topk: int = 0
    H_I: int = 0
    d_I: int = 0
    rope_dims: int = 64
    rope_base: float = 10000.0
    idx_rope_dims: int = 0
    q_idx_rope: bool = False
    eps: float = 1e-6
    softmax_scale: float = 0.0
    gamma_idx: torch.Tensor | None = None
    idx_state: DeviceState | None = None
    idx_cache: DeviceCache | None = None
    gamma_q: torch.Tensor | None = None
    _ws: torch.Tensor | None = field(default=None, repr=False)

    def struct(self) -> A.Layer:
        L = A.Layer()
        L.kind = A.LAYER_C4 if self.kind == "c4" else A.LAYER_C128
        L.heads, L.dim, L.topk, L.idx_heads, L.idx_dim = self.H, self.D, self.topk, self.H_I, self.d_I
        L.rope = A.Rope(self.rope_dims, self.rope_base)
        L.idx_rope_dims = self.idx_rope_dims
        L.q_idx_rope = int(self.q_idx_rope)
        L.eps = self.eps
        L.softmax_scale = self.softmax_scale
        L.gamma = _ptr(self.gamma)
        L.gamma_idx = _ptr(self.gamma_idx)
        L.state = self.state.struct()
        L.cache = self.cache.struct()
        L.ring = self.ring.struct()
        L.gamma_q = _ptr(self.gamma_q)
        if self.kind == "c4":
            L.idx_state = self.idx_state.struct()
            L.idx_cache = self.idx_cache.struct()
        return L

    @classmethod
    def from_arrays(cls, la, device="cuda") -> "DeviceLayer":
        """Upload a layer given as numpy byte arrays (the synthetic workload layout)."""
        s = la.spec
        dev = torch.device(device)
        f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
        layer = cls(kind=s.kind, H=s.H, D=s.D, gamma=f(la.gamma.astype(np.float32)),
                    state=DeviceState(f(la.state.astype(np.float32)), s.D),
                    cache=DeviceCache(to_device_codes(la.pages, s.cache_dtype, dev), f(la.scales),
                                      f(la.block_table.astype(np.int32)), s.m, s.cache_dtype),
                    ring=DeviceRing(to_device_codes(la.swa_rows, s.swa_dtype, dev), f(la.swa_scales), s.swa_dtype),
                    topk=s.k, H_I=s.H_I, d_I=s.d_I, rope_dims=s.rope_dims, rope_base=s.rope_base,
                    idx_rope_dims=s.idx_rope_dims, q_idx_rope=s.q_idx_rope, eps=s.eps)
        if getattr(la, "gamma_q", None) is not None:
            layer.gamma_q = f(la.gamma_q.astype(np.float32))
        if s.kind == "c4":
            layer.gamma_idx = f(la.gamma_idx.astype(np.float32))
            layer.idx_state = DeviceState(f(la.idx_state.astype(np.float32)), s.d_I)
            layer.idx_cache = DeviceCache(to_device_codes(la.idx_pages, s.idx_dtype, dev), f(la.idx_scales),
                                          f(la.idx_block_table.astype(np.int32)), s.m, s.idx_dtype)
        return layer

    def workspace_bytes(self, batch: int) -> int:
        return A.load().dsv4_hybrid_decode_workspace_size(C.byref(self.struct()), batch)

    def workspace(self, batch: int) -> torch.Tensor:
        n = self.workspace_bytes(batch)
        if self._ws is None or self._ws.numel() < n:
            self._ws = torch.empty(max(n, 256), dtype=torch.uint8, device=self.gamma.device)
        return self._ws


@dataclass
class DeviceStep:
    pos: torch.Tensor
    kv: torch.Tensor
    gate: torch.Tensor
    q: torch.Tensor
    out: torch.Tensor
    kv_dtype: str
    q_dtype: str
    out_dtype: str
    idx_kv: torch.Tensor | None = None
    idx_gate: torch.Tensor | None = None
    q_idx: torch.Tensor | None = None
    q_idx_dtype: str = "fp8"
    q_idx_scale: torch.Tensor | None = None
    w: torch.Tensor | None = None
    w_dtype: str = "bf16"
    topk_idx: torch.Tensor | None = None
    d_status: torch.Tensor | None = None
    out_scales: torch.Tensor | None = None  # [B, H, D/128] float32 for fp8 outputs

    def struct(self) -> A.Step:
        S = A.Step()
        S.batch = self.pos.shape[0]
        S.pos, S.kv, S.gate = _ptr(self.pos), _ptr(self.kv), _ptr(self.gate)
        S.idx_kv, S.idx_gate = _ptr(self.idx_kv), _ptr(self.idx_gate)
        S.kv_dtype = DT[self.kv_dtype]
        S.q, S.q_dtype = _ptr(self.q), DT[self.q_dtype]
        S.q_idx, S.q_idx_dtype = _ptr(self.q_idx), DT[self.q_idx_dtype]
        S.q_idx_scale = _ptr(self.q_idx_scale)
        S.w, S.w_dtype = _ptr(self.w), DT[self.w_dtype]
        S.out, S.out_dtype = _ptr(self.out), DT[self.out_dtype]
        S.topk_idx = _ptr(self.topk_idx)
        S.d_status = _ptr(self.d_status)
        S.out_scales = _ptr(self.out_scales)
        return S

    @classmethod
    def from_arrays(cls, spec, st, device="cuda", with_topk: bool = True) -> "DeviceStep":
        dev = torch.device(device)
        f = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev)  # noqa: E731
        c = lambda a, dt: None if a is None else to_device_codes(a, dt, dev)  # noqa: E731
        B = st.pos.shape[0]
        step = cls(pos=f(st.pos.astype(np.int32)), kv=c(st.kv, spec.kv_dtype), gate=c(st.gate, spec.kv_dtype),
                   q=c(st.q, spec.q_dtype),
                   out=torch.empty((B, spec.H, spec.D), dtype=TORCH_CODE_DTYPE[spec.out_dtype], device=dev),
                   kv_dtype=spec.kv_dtype, q_dtype=spec.q_dtype, out_dtype=spec.out_dtype,
                   d_status=torch.zeros(1, dtype=torch.int32, device=dev))
        if spec.out_dtype == "fp8":
            step.out_scales = torch.empty((B, spec.H, spec.D // A.OUT_BLOCK), dtype=torch.float32, device=dev)
        if spec.kind == "c4":
            step.idx_kv, step.idx_gate = c(st.idx_kv, spec.kv_dtype), c(st.idx_gate, spec.kv_dtype)
            step.q_idx, step.q_idx_dtype = c(st.q_idx, spec.q_idx_dtype), spec.q_idx_dtype
            step.q_idx_scale = f(st.q_idx_scale)
            step.w, step.w_dtype = c(st.w, spec.w_dtype), spec.w_dtype
            if with_topk:
                step.topk_idx = torch.empty((B, spec.k), dtype=torch.int32, device=dev)
        return step


# ---------------------------------------------------------------------------
# entry points

def hybrid_decode(layer: DeviceLayer, step: DeviceStep, workspace: torch.Tensor | None = None, stream=None):
    """One decode step of one layer (updates the layer's caches and states in place)."""
    lib = A.load()
    B = step.pos.shape[0]
    ws = workspace if workspace is not None else layer.workspace(B)
    L, S = layer.struct(), step.struct()
    A.check("dsv4_hybrid_decode",
            lib.dsv4_hybrid_decode(C.byref(L), C.byref(S), _ptr(ws), ws.numel(), _stream(stream)))
    return step.out


def compress(kv, gate, cu_seqlens, start_pos, state: DeviceState, cache: DeviceCache, gamma, *, kv_dtype: str,
             eps: float = 1e-6, rope_dims: int = 64, rope_base: float = 10000.0, d_status=None, stream=None):
    lib = A.load()
    a = A.CompressArgs(batch=cu_seqlens.shape[0] - 1, total_tokens=kv.shape[0], kv=_ptr(kv), gate=_ptr(gate),
                       kv_dtype=DT[kv_dtype], cu_seqlens=_ptr(cu_seqlens), start_pos=_ptr(start_pos),
                       gamma=_ptr(gamma), eps=eps, rope=A.Rope(rope_dims, rope_base), state=state.struct(),
                       cache=cache.struct(), d_status=_ptr(d_status))
    A.check("dsv4_compress", lib.dsv4_compress(C.byref(a), _stream(stream)))


def compress_project(hidden, w, cu_seqlens, start_pos, state: DeviceState, cache: DeviceCache, gamma, *,
                     eps: float = 1e-6, rope_dims: int = 64, rope_base: float = 10000.0, d_status=None,
                     workspace=None, stream=None):
    """dsv4_compress_project: kv, gate = bf16(hidden [T, Hd] . w [2D, Hd]^T) on the tensor cores,
    then the compressor. Returns (kv, gate): views [T, D] bf16 of the workspace, which hold
    the projection after the call."""
    lib = A.load()
    T, Hd = hidden.shape
    D = state.dim
    c = A.CompressArgs(batch=cu_seqlens.shape[0] - 1, total_tokens=T, kv=None, gate=None, kv_dtype=A.BF16,
                       cu_seqlens=_ptr(cu_seqlens), start_pos=_ptr(start_pos), gamma=_ptr(gamma), eps=eps,
                       rope=A.Rope(rope_dims, rope_base), state=state.struct(), cache=cache.struct(),
                       d_status=_ptr(d_status))
    a = A.CompressProjectArgs(c=c, hidden=_ptr(hidden), w=_ptr(w), hidden_dim=Hd)
    need = lib.dsv4_compress_project_workspace_size(C.byref(a))
    if need == 0:
        A.check("dsv4_compress_project_workspace_size", A.ERR_INVALID_ARG)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=hidden.device)
    A.check("dsv4_compress_project", lib.dsv4_compress_project(C.byref(a), _ptr(ws), ws.numel(), _stream(stream)))
    off = (T * D * 2 + 255) // 256 * 256
    kv = ws[:T * D * 2].view(torch.bfloat16).view(T, D)
    gate = ws[off:off + T * D * 2].view(torch.bfloat16).view(T, D)
    return kv, gate


def swa_insert(kv, cu_seqlens, start_pos, ring: DeviceRing, gamma, *, kv_dtype: str, eps: float = 1e-6,
               rope_dims: int = 64, rope_base: float = 10000.0, d_status=None, stream=None):
    lib = A.load()
    a = A.SwaInsertArgs(batch=cu_seqlens.shape[0] - 1, total_tokens=kv.shape[0], kv=_ptr(kv), kv_dtype=DT[kv_dtype],
                        cu_seqlens=_ptr(cu_seqlens), start_pos=_ptr(start_pos), gamma=_ptr(gamma), eps=eps,
                        rope=A.Rope(rope_dims, rope_base), ring=ring.struct(), d_status=_ptr(d_status))
    A.check("dsv4_swa_insert", lib.dsv4_swa_insert(C.byref(a), _stream(stream)))


def indexer_args(q_idx, w, keys: DeviceCache, n_entries, k: int, *, q_dtype: str, w_dtype: str, q_scale=None,
                 pos=None, q_rope_dims: int = 0, rope_base: float = 10000.0, idx=None, scores=None,
                 d_status=None) -> A.IndexerArgs:
    B, H, Dq = q_idx.shape
    return A.IndexerArgs(batch=B, heads=H, dim=Dq, k=k, q_idx=_ptr(q_idx), q_dtype=DT[q_dtype],
                         q_scale=_ptr(q_scale), w=_ptr(w), w_dtype=DT[w_dtype], keys=keys.struct(),
                         n_entries=_ptr(n_entries), pos=_ptr(pos), q_rope_dims=q_rope_dims, rope_base=rope_base,
                         idx=_ptr(idx), scores=_ptr(scores), d_status=_ptr(d_status))


def indexer_topk(q_idx, w, keys: DeviceCache, n_entries, k: int, *, q_dtype: str, w_dtype: str, q_scale=None,
                 pos=None, q_rope_dims: int = 0, rope_base: float = 10000.0, with_scores: bool = True,
                 d_status=None, workspace=None, stream=None):
    """Top-k entry indices [B, k] (and their scores) of the lightning indexer."""
    lib = A.load()
    B = q_idx.shape[0]
    idx = torch.empty((B, k), dtype=torch.int32, device=q_idx.device)
    scores = torch.empty((B, k), dtype=torch.float32, device=q_idx.device) if with_scores else None
    a = indexer_args(q_idx, w, keys, n_entries, k, q_dtype=q_dtype, w_dtype=w_dtype, q_scale=q_scale, pos=pos,
                     q_rope_dims=q_rope_dims, rope_base=rope_base, idx=idx, scores=scores, d_status=d_status)
    need = lib.dsv4_indexer_workspace_size(C.byref(a))
    if need == 0:
        A.check("dsv4_indexer_workspace_size", A.ERR_INVALID_ARG)
    ws = workspace if workspace is not None else torch.empty(need, dtype=torch.uint8, device=q_idx.device)
    A.check("dsv4_indexer_topk", lib.dsv4_indexer_topk(C.byref(a), _ptr(ws), ws.numel(), _stream(stream)))
    return idx, scores


def indexer_scores(q_idx, w, keys: DeviceCache, n_entries, *, q_dtype: str, w_dtype: str, q_scale=None, out=None,
                   d_status=None, stream=None):
    """Every visible entry's indexer score, [B, ld] float32 (ld = the cache capacity rounded up
    to 4); entries past n_entries are left as `out` held them."""
    B = q_idx.shape[0]
    cap = keys.block_table.shape[1] * (A.PAGE_POSITIONS // keys.m)
    ld = (cap + 3) // 4 * 4
    if out is None:
        out = torch.full((B, ld), float("nan"), dtype=torch.float32, device=q_idx.device)
    a = indexer_args(q_idx, w, keys, n_entries, 1, q_dtype=q_dtype, w_dtype=w_dtype, q_scale=q_scale,
                     d_status=d_status)
    A.check("dsv4_indexer_scores", A.load().dsv4_indexer_scores(C.byref(a), _ptr(out), out.shape[1], _stream(stream)))
    return out


def indexer_topk_noalloc(q_idx, w, keys: DeviceCache, n_entries, k: int, *, idx, q_dtype: str, w_dtype: str,
                         scores=None, q_scale=None, pos=None, q_rope_dims: int = 0, rope_base: float = 10000.0,
                         d_status=None, stream=None):
    """indexer_topk on the library's static scratch: the caller passes the outputs (idx [B, k]
    int32, optionally scores [B, k] float32) and nothing is allocated by this call."""
    a = indexer_args(q_idx, w, keys, n_entries, k, q_dtype=q_dtype, w_dtype=w_dtype, q_scale=q_scale, pos=pos,
                     q_rope_dims=q_rope_dims, rope_base=rope_base, idx=idx, scores=scores, d_status=d_status)
    A.check("dsv4_indexer_topk_noalloc", A.load().dsv4_indexer_topk_noalloc(C.byref(a), _stream(stream)))
    return idx, scores


def mqa_args(q, pos, cache: DeviceCache, ring: DeviceRing, *, q_dtype: str, out, out_dtype: str, idx=None,
             n_entries=None, softmax_scale: float = 0.0, rope_dims: int = 64, rope_base: float = 10000.0, lse=None,
             d_status=None, q_norm_gamma=None, q_norm_eps: float = 1e-6, out_scales=None) -> A.MqaArgs:
    B, H, D = q.shape
    return A.MqaArgs(batch=B, heads=H, dim=D, q=_ptr(q), q_dtype=DT[q_dtype], pos=_ptr(pos), cache=cache.struct(),
                     n_entries=_ptr(n_entries), idx=_ptr(idx), k=0 if idx is None else idx.shape[1],
                     ring=ring.struct(), softmax_scale=softmax_scale, rope=A.Rope(rope_dims, rope_base),
                     out=_ptr(out), out_dtype=DT[out_dtype], lse=_ptr(lse), d_status=_ptr(d_status),
                     q_norm_gamma=_ptr(q_norm_gamma), q_norm_eps=q_norm_eps, out_scales=_ptr(out_scales))


def mqa_workspace_size(args: A.MqaArgs) -> int:
    """dsv4_mqa_workspace_size for the marshalled arguments of a sparse_mqa_decode call."""
    return A.load().dsv4_mqa_workspace_size(C.byref(args))


def sparse_mqa_decode(q, pos, cache: DeviceCache, ring: DeviceRing, *, q_dtype: str, out_dtype: str, idx=None,
                      n_entries=None, softmax_scale: float = 0.0, rope_dims: int = 64, rope_base: float = 10000.0,
                      with_lse: bool = False, d_status=None, workspace=None, stream=None, q_norm_gamma=None,
                      q_norm_eps: float = 1e-6):
    """Returns out (and lse); for fp8 outputs, out is (codes, scales [B, H, D/128])."""
    lib = A.load()
    B, H, D = q.shape
    out = torch.empty((B, H, D), dtype=TORCH_CODE_DTYPE[out_dtype], device=q.device)
    out_scales = (torch.empty((B, H, D // A.OUT_BLOCK), dtype=torch.float32, device=q.device)
                  if out_dtype == "fp8" else None)
    lse = torch.empty((B, H), dtype=torch.float32, device=q.device) if with_lse else None
    a = mqa_args(q, pos, cache, ring, q_dtype=q_dtype, out=out, out_dtype=out_dtype, idx=idx, n_entries=n_entries,
                 softmax_scale=softmax_scale, rope_dims=rope_dims, rope_base=rope_base, lse=lse, d_status=d_status,
                 q_norm_gamma=q_norm_gamma, q_norm_eps=q_norm_eps, out_scales=out_scales)
    need = lib.dsv4_mqa_workspace_size(C.byref(a))
    ws = workspace if workspace is not None else torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    A.check("dsv4_sparse_mqa_decode", lib.dsv4_sparse_mqa_decode(C.byref(a), _ptr(ws), ws.numel(), _stream(stream)))
    res = (out, out_scales) if out_dtype == "fp8" else out
    return (res, lse) if with_lse else res


def layer_state_bytes(context: int, m: int, entry_width: int, window: int, window_width: int,
                      bytes_per_value: int) -> int:
    return A.load().dsv4_layer_state_bytes(context, m, entry_width, window, window_width, bytes_per_value)
