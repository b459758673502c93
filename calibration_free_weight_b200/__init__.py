"""HQQ zero-point solver for NVIDIA B200 (sm_100a): C-ABI library + thin binding.

``calibration_free_weight_b200.hqq`` binds ``libhqq_b200.so`` (include/hqq.h);
``calibration_free_weight_b200.synth`` generates seeded synthetic weights.
The binding is imported on first attribute access so that input generation
does not need the CUDA library; using the binding without the library raises.
"""
import importlib


def __getattr__(name):
    if name == "hqq":
        return importlib.import_module(__name__ + ".hqq")
    raise AttributeError(name)
