"""B200-native FFN-pool expert layer of attention-FFN disaggregation (AFD).

The layer (C ABI in include/afd_ffn.h, CUDA in csrc/) takes block-FP8 tokens and top-K
routing that M attention ranks published into receive slabs on this GPU, runs the routed
experts as tcgen05 FP8 grouped GEMMs with SwiGLU between them, and writes each token's
top-K-weighted bf16 result back into its slab row. `ffn` is the ctypes binding.
"""
from .ffn import FfnLayer, AfdError, lib, kernels_per_layer, check_config, make_config  # noqa: F401
