"""Layer-streamed NF4 QLoRA training on B200 (sm_100a).

Modules: ``binding`` (ctypes view of libnf4ls.so), ``api`` (the same calls with torch
buffers), ``synth`` (seeded synthetic inputs), ``build`` (nvcc build of the library),
``steplog`` (per-step JSON-lines log of a training run).
Importing the package loads nothing; the library loads on first use.
"""
__all__ = ["api", "binding", "synth", "build", "steplog"]
