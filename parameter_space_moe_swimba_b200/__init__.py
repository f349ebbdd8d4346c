"""Swimba (Switch Mamba) layer on B200: a C-ABI library of sm_100a CUDA kernels.

``parameter_space_moe_swimba_b200.swimba`` is the ctypes binding of ``libswimba.so`` (imported on
demand, so the shape tables and the synthetic-input generator work without a GPU or a build).
"""
from . import configs, synth  # noqa: F401

__all__ = ["configs", "synth"]
