"""ctypes mirror of include/dsv4.h (argument marshalling only)."""

from __future__ import annotations

import ctypes as C
import os

from .build import LIB

F32, BF16, FP8, FP4 = 0, 1, 2, 3
LAYER_C4, LAYER_C128 = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_SCRATCH_LIMIT = 0, 1, 2, 3, 4
NOALLOC_SCRATCH_BYTES = 16 << 20
DEV_BAD_INDEX, DEV_BAD_PAGE, DEV_TIMEOUT, DEV_BAD_LENGTH = 1, 2, 4, 8
PAGE_POSITIONS = 256
OUT_BLOCK = 128  # channels per fp8 output block

DTYPE_CODE = {"f32": F32, "bf16": BF16, "fp8": FP8, "fp4": FP4}

p = C.c_void_p
i32 = C.c_int32


class Rope(C.Structure):
    _fields_ = [("rope_dims", i32), ("rope_base", C.c_float)]


class PagedCache(C.Structure):
    _fields_ = [("pages", p), ("scales", p), ("block_table", p), ("num_pages", i32), ("max_blocks", i32),
                ("dim", i32), ("m", i32), ("dtype", C.c_int)]


class WindowRing(C.Structure):
    _fields_ = [("rows", p), ("scales", p), ("window", i32), ("dim", i32), ("dtype", C.c_int)]


class CompressorState(C.Structure):
    _fields_ = [("buf", p), ("m", i32), ("dim", i32), ("gate_dim", i32)]


class CompressArgs(C.Structure):
    _fields_ = [("batch", i32), ("total_tokens", i32), ("kv", p), ("gate", p), ("kv_dtype", C.c_int),
                ("cu_seqlens", p), ("start_pos", p), ("gamma", p), ("eps", C.c_float), ("rope", Rope),
                ("state", CompressorState), ("cache", PagedCache), ("d_status", p)]


class CompressProjectArgs(C.Structure):
    _fields_ = [("c", CompressArgs), ("hidden", p), ("w", p), ("hidden_dim", i32)]


class SwaInsertArgs(C.Structure):
    _fields_ = [("batch", i32), ("total_tokens", i32), ("kv", p), ("kv_dtype", C.c_int), ("cu_seqlens", p),
                ("start_pos", p), ("gamma", p), ("eps", C.c_float), ("rope", Rope), ("ring", WindowRing),
                ("d_status", p)]


class IndexerArgs(C.Structure):
    _fields_ = [("batch", i32), ("heads", i32), ("dim", i32), ("k", i32), ("q_idx", p), ("q_dtype", C.c_int),
                ("q_scale", p), ("w", p), ("w_dtype", C.c_int), ("keys", PagedCache), ("n_entries", p),
                ("pos", p), ("q_rope_dims", i32), ("rope_base", C.c_float), ("idx", p), ("scores", p),
                ("d_status", p)]


class MqaArgs(C.Structure):
    _fields_ = [("batch", i32), ("heads", i32), ("dim", i32), ("q", p), ("q_dtype", C.c_int), ("pos", p),
                ("cache", PagedCache), ("n_entries", p), ("idx", p), ("k", i32), ("ring", WindowRing),
                ("softmax_scale", C.c_float), ("rope", Rope), ("out", p), ("out_dtype", C.c_int), ("lse", p),
                ("d_status", p), ("q_norm_gamma", p), ("q_norm_eps", C.c_float), ("out_scales", p)]


class Layer(C.Structure):
    _fields_ = [("kind", C.c_int), ("heads", i32), ("dim", i32), ("topk", i32), ("idx_heads", i32),
                ("idx_dim", i32), ("rope", Rope), ("idx_rope_dims", i32), ("q_idx_rope", i32),
                ("eps", C.c_float), ("softmax_scale", C.c_float), ("gamma", p), ("gamma_idx", p),
                ("state", CompressorState), ("cache", PagedCache), ("ring", WindowRing),
                ("idx_state", CompressorState), ("idx_cache", PagedCache), ("gamma_q", p)]


class Step(C.Structure):
    _fields_ = [("batch", i32), ("pos", p), ("kv", p), ("gate", p), ("idx_kv", p), ("idx_gate", p),
                ("kv_dtype", C.c_int), ("q", p), ("q_dtype", C.c_int), ("q_idx", p), ("q_idx_dtype", C.c_int),
                ("q_idx_scale", p), ("w", p), ("w_dtype", C.c_int), ("out", p), ("out_dtype", C.c_int),
                ("topk_idx", p), ("d_status", p), ("out_scales", p)]


EXPORTS = {
    "dsv4_compress": (C.c_int, [C.POINTER(CompressArgs), p]),
    "dsv4_compress_project_workspace_size": (C.c_size_t, [C.POINTER(CompressProjectArgs)]),
    "dsv4_compress_project": (C.c_int, [C.POINTER(CompressProjectArgs), p, C.c_size_t, p]),
    "dsv4_swa_insert": (C.c_int, [C.POINTER(SwaInsertArgs), p]),
    "dsv4_indexer_workspace_size": (C.c_size_t, [C.POINTER(IndexerArgs)]),
    "dsv4_indexer_topk": (C.c_int, [C.POINTER(IndexerArgs), p, C.c_size_t, p]),
    "dsv4_indexer_topk_noalloc": (C.c_int, [C.POINTER(IndexerArgs), p]),
    "dsv4_indexer_scores": (C.c_int, [C.POINTER(IndexerArgs), p, C.c_int64, p]),
    "dsv4_mqa_workspace_size": (C.c_size_t, [C.POINTER(MqaArgs)]),
    "dsv4_sparse_mqa_decode": (C.c_int, [C.POINTER(MqaArgs), p, C.c_size_t, p]),
    "dsv4_hybrid_decode_workspace_size": (C.c_size_t, [C.POINTER(Layer), i32]),
    "dsv4_hybrid_decode": (C.c_int, [C.POINTER(Layer), C.POINTER(Step), p, C.c_size_t, p]),
    "dsv4_status_string": (C.c_char_p, [C.c_int]),
    "dsv4_abi_version": (i32, []),
    "dsv4_launch_count": (C.c_uint64, []),
    "dsv4_layer_state_bytes": (C.c_uint64, [C.c_uint64, i32, i32, i32, i32, i32]),
}

_lib = None


def load() -> C.CDLL:
    """Load the in-tree libdsv4.so; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} is missing: build it with `python -m compressed_sparse_kv_dsv4_b200.build`")
        lib = C.CDLL(LIB)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class Dsv4Error(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = load().dsv4_status_string(code).decode()
        super().__init__(f"{fn}: {msg} ({code})")
        self.code = code


def check(fn: str, code: int) -> None:
    if code != OK:
        raise Dsv4Error(fn, code)
