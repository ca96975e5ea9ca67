"""B200-native single-GPU core of an expert-parallel MoE layer.

route top-k -> dispatch layout -> permute (optional FP8 payload) ->
grouped SwiGLU expert GEMM -> weighted combine, each step a call into the
C-ABI library ``libmoe.so`` built from ``csrc/``.  ``workloads`` and
``traffic`` are host-only helpers and import without the library; the
binding (``expert_parallelism_b200.moe``) loads the library on first use
and raises if it is missing.
"""
__all__ = ["workloads", "traffic"]
