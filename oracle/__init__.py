"""Independent fp64 CPU oracle for GQA prefill/decode (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline / reference
leg may import this package.  The product library never uses it.
"""
from .gqa_ref import (  # noqa: F401
    as_f64, head_group, inv_freq, rope, rope_interleaved, softmax_rows, causal_weights,
    prefill_ref, prefill_rows_ref, decode_one_ref, decode_ref, packed_offsets,
    prefill_flops, decode_bytes,
)
