"""Block top-k sparse attention decode over a paged KV cache, for B200 (sm_100a).

The compute lives in the C-ABI library libvx.so (hand-written CUDA, see include/vx.h);
the Python side only marshals arguments.  `synth` draws seeded synthetic workloads.
"""
