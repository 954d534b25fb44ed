"""B200-native fused sigmoid-gating Gated DeltaNet decode update.

The product is the C-ABI library ``libgdn_decode.so`` (declared in
``include/gdn_decode.h``), whose sm_100a kernel performs the whole decode /
speculative-decode state update.  ``binding`` is a thin ctypes layer that
marshals torch tensors into that ABI; ``workloads`` draws seeded synthetic
inputs.  The binding loads the library on first use and raises if it is
missing: there is no CPU or library fallback.
"""
from __future__ import annotations

__all__ = ["decode_update", "recurrent_update", "gating", "binding", "workloads"]


def __getattr__(name):
    # Lazy: importing the package (e.g. for ``workloads``) must not need the
    # CUDA library; calling into it must.
    if name in ("decode_update", "decode_update_host", "recurrent_update", "gating", "PreparedCall",
                "HostStagedDecode", "GdnError", "L2NORM_QK", "WRITE_INTERMEDIATE", "NO_FINAL_WRITEBACK",
                "CHECK_INDICES", "LAUNCH_PDL"):
        from . import binding
        return getattr(binding, name)
    if name in ("binding", "workloads", "build"):
        import importlib
        return importlib.import_module(f"{__name__}.{name}")
    raise AttributeError(name)
