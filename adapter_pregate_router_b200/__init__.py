"""Token-level pre-gated mixture-of-LoRA with segmented gather products on B200.

The compute path is ``libapr.so`` (CUDA, sm_100a) behind a C ABI declared in
``include/apr.h``; ``adapter_pregate_router_b200.apr`` is its Python binding.
Importing the package itself loads nothing, so ``workloads`` can be used
without the library.
"""

__all__ = ["apr", "workloads"]
