"""Quantized Delta-rule recurrent-state decode step for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library built from ``csrc/`` (``libstq.so``);
``binding`` is a thin ctypes layer over it and ``workloads`` holds the seeded
synthetic inputs.  Importing the package loads nothing; ``binding.lib()``
loads the CUDA library and raises if it is missing.
"""
__all__ = ["binding", "workloads"]
