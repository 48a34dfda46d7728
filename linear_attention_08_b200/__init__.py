"""Kimi Delta Attention (KDA) on B200: chunked prefill, state checkpoints, decode.

The operator runs in hand-written sm_100a CUDA kernels behind the C ABI in
include/kda.h (libkda.so, built in-tree by ``linear_attention_08_b200.build``).
``linear_attention_08_b200.kda`` is the ctypes binding; ``inputs`` draws the
seeded synthetic workloads.
"""
from .kda import (kda_ckpt_count, kda_decode, kda_decode_multi,  # noqa: F401
                  kda_prefill, kda_prefill_path, kda_selftest_bounded_wait, load)

__version__ = "0.1.0"
