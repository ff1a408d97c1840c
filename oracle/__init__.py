"""fp64 CPU oracle for Heavily Compressed Attention (HCA): the forward in plain C
(compress, prefill rows, decode), Virtual Head Attention and the backward pass in numpy,
and the sparse-attention layers' indexer / top-k / core attention decode step in numpy.

TEST INFRASTRUCTURE ONLY.  Only tests/, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with
the CUDA library in ``compressed_long_context_b200``.
"""
from .oracle import (  # noqa: F401
    compress, round_bf16, visible_entries, prefill_rows, decode, num_threads,
    bf16_bits, bits_to_f64, vha, gate_logits,
)
from . import backward  # noqa: F401  (fp64 gradients of the layer, numpy)
from . import dsa  # noqa: F401  (indexer, top-k selection and sparse attention, numpy)
