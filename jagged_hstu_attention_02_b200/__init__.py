"""Jagged HSTU attention for B200 (sm_100a).

The compute path lives in the CUDA shared library built from csrc/ (C-ABI declared in
include/hstu_attn.h).  `ops` is its thin Python binding; `synth` draws seeded inputs and
`accounting` counts valid pairs, FLOPs and bytes.  Nothing here computes the method on
the CPU: without the built library (or without a GPU) the binding raises.
"""
__all__ = ["ops", "synth", "accounting", "shard", "mfalcon"]
