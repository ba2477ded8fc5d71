"""aq: tile-aligned mixed W4/W8 x A8 linear layers for NVIDIA B200 (sm_100a).

The compute lives in libaq.so (hand-written CUDA behind a C ABI, see
include/aq.h); ``w8_a8_quantized_b200.aq`` is its thin Python binding and
``w8_a8_quantized_b200.synth`` draws seeded synthetic inputs.
"""
