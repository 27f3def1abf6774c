"""B200-native multi-scale retention forward.

The compute lives in ``libretention.so`` (hand-written sm_100a CUDA behind a
C ABI, declared in ``include/retention.h``).  ``retention`` is a thin ctypes
binding with the same entry-point names; it is imported on first use so that
the input generator (``synth``) can be used without the library.
"""
from importlib import import_module

_BINDING_NAMES = (
    "ret_parallel", "ret_chunkwise", "ret_chunkwise_gate_static", "ret_recurrent_step",
    "ret_gate_norm",
    "ret_workspace_size", "ret_last_device_status", "ret_kernel_launches",
    "ret_status_string",
    "RetentionError", "msr_gammas", "load_library",
)


def __getattr__(name):
    if name in _BINDING_NAMES:
        return getattr(import_module(".retention", __name__), name)
    raise AttributeError(name)
