"""B200-native (sm_100a) selective state-space scan.

The CUDA library (``libssm_scan_b200.so``, C ABI in ``include/ssm_scan.h``)
does all of the scan's work; this package only marshals arguments to it.
Importing the package does not load the library: the first call that needs
it does, and fails loudly if it is missing.
"""
from __future__ import annotations

__all__ = ["fwd", "step", "direct", "Plan", "load_library", "SsmError"]


def __getattr__(name):
    if name in __all__:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
