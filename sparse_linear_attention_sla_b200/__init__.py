"""B200-native (sm_100a) SLA / SLA2 sparse-plus-linear block attention forward.

The computation lives in libsla.so (CUDA kernels behind the C ABI of
include/sla.h). ``sparse_linear_attention_sla_b200.binding`` is the thin torch
binding (``forward``, ``route``, ``kv_states``); ``workloads`` draws the seeded
synthetic inputs. Importing the package loads nothing; the library is loaded
on first use of the binding.
"""

__version__ = "0.1.0"

_BINDING_NAMES = ("forward", "route", "kv_states", "check", "counts", "problem", "new_workspace",
                  "workspace_size", "version", "SlaError")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding

        return getattr(binding, name)
    raise AttributeError(name)
