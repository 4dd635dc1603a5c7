"""CPU oracle for one sparse mixture-of-experts layer forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import this package.  The CUDA
library never calls it and shares no code with it; the two meet only through the
seeded input generator ``moe_inputs``.

Everything here is plain numpy in float64, written to be read against the
pages it follows, not to be fast:

* ``formats``  - exact decoders of the expert storage formats (bf16, MXFP4,
  NVFP4, INT4 group-128), from the format definitions the pages name
  ("Mixture of experts VRAM: total vs active parameters", section "How current
  MoE models route each token": FP4 and INT4 experts; "Understanding MoE
  Inference Costs on Galactus", August table: MXFP4 and native-INT4 experts).
* ``layer``    - router, softmax/top-k with renormalisation, the stable
  per-expert permutation, the SwiGLU expert FFN, the weighted combine and the
  shared expert; plus the per-token routing margin and the fp32 rounding bound
  used to decide which tokens' expert choice is unique.
* ``lru``      - an exact replay of the per-layer LRU expert cache.

Pins (``tests/test_oracle_*.py``) tie each function to something other than
itself: spec tables and library decoders for the formats, brute force over all
k-subsets for top-k, a library stable sort for the permutation, closed forms
and invariants for the FFN and combine, and a hand-worked trace for the LRU.
"""
