"""B200-native MoE layer forward: router, hash gate, dispatch, grouped SwiGLU experts, combine.

The compute lives in the CUDA library ``libmoe.so`` (sources under ``csrc/``),
reached through a plain C ABI.  ``mixture_experts_routing_gate_b200.moe``
is the thin Python binding (argument marshalling only); importing it fails
loudly when the library has not been built.  ``workloads`` draws the seeded
synthetic layers used by the tests and the benchmark.
"""
__all__ = ["moe", "workloads"]
