"""CPR Gated DeltaNet on B200: a C-ABI CUDA library (libgdn_cpr.so) and its binding.

``rl_train_numerics_b200.gdn`` is the Python binding (imported lazily, since
it loads the CUDA library); ``rl_train_numerics_b200.workloads`` draws the
seeded synthetic inputs.
"""
import importlib

__all__ = ["gdn", "workloads", "build_lib"]


def __getattr__(name):
    if name == "gdn":
        return importlib.import_module("rl_train_numerics_b200._abi")
    if name in ("workloads", "build_lib"):
        return importlib.import_module(f"rl_train_numerics_b200.{name}")
    raise AttributeError(name)
