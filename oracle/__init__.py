"""fp64 CPU oracle for the Gated DeltaNet mixer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package.  The CUDA product path never does.
"""
from .oracle import build, prefill, decode, core, state_map, PrefillResult, default_threads, silu, gated_rmsnorm, layer, LayerResult, bf16  # noqa: F401
