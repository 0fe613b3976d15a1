"""E2D2 fused block-diffusion attention for NVIDIA B200 (sm_100a).

The attention calls of "Encoder-Decoder Diffusion Language Models for Efficient Training and
Inference" (block-causal encoder self-attention; decoder fused self+cross attention in training
and sampling mode; KV-cache append) as hand-written tcgen05/TMA kernels behind a C ABI
(include/e2d2_attn.h).  ``attn`` is the torch-tensor front-end; ``synth`` and ``workloads``
hold the seeded synthetic inputs and workload shapes.
"""
from . import synth, workloads  # noqa: F401

__all__ = ["attn", "synth", "workloads"]
