"""Paged-KV long-history causal GQA prefill attention for B200 (sm_100a).

The compute path is the C-ABI library ``libpa.so`` (CUDA kernels for sm_100a); the Python
functions in ``paged_kv_long_b200.binding`` only marshal arguments into it. Importing the
package loads nothing; the first call into the binding loads the library and raises if it is
missing. ``paged_kv_long_b200.inputs`` (seeded synthetic inputs) needs no library at all.
"""

_BINDING_NAMES = ("Plan", "PaError", "combine", "device_error", "lib_path", "load_library", "plan",
                  "prefill", "prefill_combine")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
