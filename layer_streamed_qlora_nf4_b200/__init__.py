"""Layer-streamed QLoRA (NF4) for B200: a C-ABI CUDA library plus a thin binding.

Importing the package loads nothing; ``layer_streamed_qlora_nf4_b200.lib`` loads
the compiled library on first use and fails loudly if it is missing.
"""

__all__ = ["synth", "lib"]
