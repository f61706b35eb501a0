"""liblora_sgmv for B200: the multi-adapter LoRA chunked-SGMV shrink/expand pair.

The compute path is the CUDA library ``liblora_sgmv.so`` (built in-tree by
``python -m scatter_gemm_b200.build``); :mod:`scatter_gemm_b200.lora` is a
thin ctypes binding over its C ABI (``include/lora_sgmv.h``).  The binding is
imported lazily so that the seeded input generators in
:mod:`scatter_gemm_b200.workloads` can be used without the CUDA library.
"""

__all__ = ["lora_shrink", "lora_expand", "lora_validate", "make_workspace",
           "workspace_size", "LoraError"]


def __getattr__(name):
    if name in __all__:
        from . import lora
        return getattr(lora, name)
    raise AttributeError(name)
