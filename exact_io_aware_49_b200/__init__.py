"""Exact, IO-aware attention for B200 (sm_100a).

The compute lives in ``libfa_sm100.so`` (hand-written CUDA, C ABI declared in
``include/fa.h``); ``binding`` marshals torch tensors into that ABI.  Importing
the package does not load the library; the first use of an entry point does,
and fails loudly if the library is missing -- there is no fallback path.
"""

_BINDING_NAMES = ("fa_fwd", "fa_bwd", "fa_fwd_varlen", "fa_bwd_varlen", "fa_decode_paged", "fa_bwd_stages",
                  "fa_bwd_workspace_size", "fa_fwd_bwd_host", "fa_fwd_bwd_host_workspace_size",
                  "fa_dropout_mask", "fa_last_device_error", "fa_selftest_wait_timeout", "FAError", "load_library")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)


__all__ = list(_BINDING_NAMES)
