"""DeltaLog deferred-materialisation decode step for linear-attention state on B200.

``DeltaLog`` (PyTorch tensors in, CUDA library underneath) and the raw C-ABI
binding ``_native`` are the public surface.  Importing this package does not
load the CUDA library; the first handle does, and fails loudly if it is
missing.
"""
__all__ = ["DeltaLog", "DeltaLogError", "suggest_m"]


def __getattr__(name):
    if name == "DeltaLog":
        from .deltalog import DeltaLog
        return DeltaLog
    if name == "suggest_m":
        from .deltalog import suggest_m
        return suggest_m
    if name == "DeltaLogError":
        from ._native import DeltaLogError
        return DeltaLogError
    raise AttributeError(name)
