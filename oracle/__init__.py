"""ORACLE — test infrastructure only.

A plain fp64 CPU statement of exact paged GQA decode attention and of the
split log-sum-exp merge, written from the source pages and kept independent
of the CUDA library (no shared code, headers or constants).  Only the tests,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
it; the product path never does.
"""
from .oracle import decode, decode_varlen, combine, append_kv, f16_to_double, bf16_to_double, library_path  # noqa: F401
