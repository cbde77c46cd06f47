"""Stem block-sparse causal prefill for NVIDIA B200 (sm_100a).

The compute lives in libstem.so (CUDA kernels behind the C ABI of include/stem.h); the names
below are its thin Python binding, loaded on first use. `workloads` holds the seeded synthetic
inputs and imports nothing from the binding.
"""

_BINDING = ("stem_prefill", "stem_prefill_ex", "stem_prefill_host", "stem_budget",
            "stem_sel_capacity", "stem_workspace_size", "stem_pool", "stem_select",
            "stem_sparse_attn", "StemError", "strerror")


def __getattr__(name):
    if name in _BINDING:
        from . import stem as _stem
        return getattr(_stem, name)
    raise AttributeError(name)


__all__ = list(_BINDING)
