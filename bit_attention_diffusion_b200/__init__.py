"""VC-Attention FP8 for B200 (sm_100a): a C-ABI CUDA library plus a thin Python binding.

The binding (``bit_attention_diffusion_b200.vcattn``) loads the in-tree shared
library ``libvcattn.so`` and fails loudly if it is missing; there is no CPU
fallback. ``synth`` draws the seeded synthetic inputs used by tests and bench.
"""
__all__ = ["synth", "vcattn"]
