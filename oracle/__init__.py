"""CPU oracle for layer-streamed QLoRA (NF4): test infrastructure, not product code.

This package is a plain, slow, obviously-correct restatement of what the hot path
computes, written from the method's description on the pages about "Exact Layer
Streaming" (the Soup layer-streaming tutorial, section "Soup layer streaming 的四段
資料路徑", parts 1-3; the Soup README, section "Retracted in v3").  It exists only
so that the CUDA library can be checked against it.

Rules it follows:
  * Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
    ``bench.py`` may import it.  The product path never calls it.
  * It shares no code, tables or constant generators with the CUDA library and
    never imports it.  Inputs come from the seeded generators in
    ``layer_streamed_qlora_nf4_b200.synth`` (which hold none of the method's
    arithmetic) or from the tests themselves.
  * Floating point is fp64, except where a floating-point result decides an
    integer (the NF4 code choice): that decision is taken in fp32, the precision
    the kernel uses, and the dequantised weight is the fp32 product
    ``level * absmax`` by definition.

Every function is pinned by ``tests/test_oracle_*.py`` against something other
than itself (closed forms, invariants, brute force, finite differences, torch
autograd and the HF transformers Llama layer).  Nothing here is "parity
unpinned".
"""

from . import nf4, model  # noqa: F401
