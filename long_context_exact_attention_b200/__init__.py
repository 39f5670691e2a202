"""Exact long-context attention for NVIDIA B200 (sm_100a).

The computation lives in the CUDA library ``liblca.so`` (C ABI in
``include/lca.h``); ``lca`` is its Python binding over torch tensors and
``inputs`` the seeded synthetic workloads.  The binding is loaded lazily so
that ``inputs`` can be imported without it; any attention call without the
built library raises.
"""

_BINDING = ("attn_fwd", "attn_bwd", "s2attn_fwd", "s2attn_bwd", "lse_merge", "check",
            "workspace_size", "LcaError", "lib")


def __getattr__(name):
    if name in _BINDING:
        from . import lca
        return getattr(lca, name)
    raise AttributeError(name)


__all__ = list(_BINDING)
