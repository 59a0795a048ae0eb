"""Causal GQA attention with a learned, input-dependent relative-position bias,
for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library ``librelbias_attn.so`` (CUDA kernels in
``csrc/``, declared in ``include/relbias_attn.h``).  ``ops`` is the thin Python
binding over it: it marshals torch tensors (device memory and streams only) into
the C calls.  ``synth`` and ``workloads`` produce the seeded synthetic inputs.

Submodules are imported lazily, so importing the package does not load CUDA.
"""
import importlib

__all__ = ["ops", "synth", "workloads", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module("." + name, __name__)
    raise AttributeError(name)
