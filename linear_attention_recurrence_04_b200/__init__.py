"""Gated DeltaNet recurrent-state update on B200 (sm_100a).

The compute lives in ``libgdn.so`` (hand-written CUDA kernels behind a C ABI,
declared in ``include/gdn.h``). ``gdn`` is the thin ctypes binding that passes
torch device tensors to it; it loads the library on first use and raises if
the library is missing: there is no CPU fallback. ``inputs`` draws the seeded
synthetic workloads and needs neither the library nor a GPU.
"""
_BINDING = ("GdnError", "step", "prefill", "pair", "layer_decode", "layer_pair", "linear_bf16",
            "forward_batch", "forward_batch_workspace_size", "forward_batch_noalloc",
            "short_conv_forward", "short_conv_forward_batch", "short_conv_pair",
            "short_conv_workspace_size", "kda_step", "kda_prefill", "library_path",
            "status_string")


def __getattr__(name):
    if name in _BINDING:
        from . import gdn
        return getattr(gdn, name)
    raise AttributeError(name)


__all__ = list(_BINDING)
