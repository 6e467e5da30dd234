"""B200-native sparse-MoE FFN step: router top-k, token grouping through an
expert-slot table, 2/3-bit SwiGLU experts with fused dequantisation, combine.

The compute lives in libmoe.so (hand-written sm_100a CUDA behind a C ABI);
`bit_expert_ffn_router_b200.moe` is its thin ctypes binding. Importing the
package loads nothing; the library is opened on first use.
"""
__all__ = ["moe", "synth"]
