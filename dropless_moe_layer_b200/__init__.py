"""Multi-round dropless MoE layer forward for NVIDIA B200 (sm_100a).

The layer routes each token to its top-k experts and runs the (token, expert)
pairs in rounds of dispatch -> grouped SwiGLU expert GEMMs -> combine, each round
with a fixed per-expert capacity C, so the layer's memory depends on its shape only
and no token is ever dropped. All compute runs in the hand-written CUDA kernels of
libmoe.so (C ABI: include/moe.h); `moe` is its Python binding.

Importing this package does not load the library; `moe.load_library()` (called by
every entry point) does, and raises if it has not been built.
"""
__all__ = ["moe", "workloads", "build"]
