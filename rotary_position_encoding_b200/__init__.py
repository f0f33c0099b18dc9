"""Fused QK-RMSNorm + causal 3D RoPE + KV-cache append for NVIDIA B200 (sm_100a).

The compute path is the CUDA library ``librope3d.so`` behind the C ABI declared in
``include/rope3d.h``; ``rope3d`` is its thin ctypes binding (argument marshalling only).
Importing this package does not load the library; the first call into ``rope3d`` does,
and raises if the library has not been built.
"""
__all__ = ["rope3d", "workloads"]
