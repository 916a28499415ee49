"""Oracle for the DeepSeek-V4 hybrid-attention decode step (test infrastructure).

A plain, slow, float64 CPU restatement of what the hot path computes. Only the
tests, the smoke check in ``__graft_entry__`` and the CPU-baseline / reference
arm of ``bench.py`` may import it; the product path (the CUDA library and its
binding) never does, and this package imports nothing from the product.
"""

from .dsv4_oracle import *  # noqa: F401,F403
