"""B200 (sm_100a) library for the DeepSeek-V4 hybrid-attention decode step.

The compute lives in libdsv4.so (CUDA kernels behind the C ABI of include/dsv4.h);
this package is its thin Python binding over torch CUDA tensors.
"""

from .binding import (DeviceCache, DeviceLayer, DeviceRing, DeviceState, DeviceStep, compress,  # noqa: F401
                      compress_project,
                      hybrid_decode, indexer_args, indexer_scores, indexer_topk, indexer_topk_noalloc,
                      layer_state_bytes, mqa_args, mqa_workspace_size, sparse_mqa_decode, swa_insert,
                      to_device_codes, to_numpy_codes)
from ._abi import Dsv4Error, load  # noqa: F401
