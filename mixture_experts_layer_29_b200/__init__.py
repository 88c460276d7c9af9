"""B200-native (sm_100a) forward pass of a LongCat-Flash Mixture-of-Experts layer.

The layer's router picks the top-K experts per token from a pool of SwiGLU FFN experts
and zero-computation (identity) experts. The work runs in hand-written CUDA kernels
behind a C ABI (include/moe.h); `mixture_experts_layer_29_b200.abi` is the Python
binding and `workloads` draws seeded synthetic inputs. Importing the package does not
load the CUDA library; `abi.lib()` does, and fails loudly when it is missing.
"""
__all__ = ["abi", "workloads"]
