"""CPU oracle for the W4A16 group-32 path.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import this package.  The product path never calls it; the CUDA
library shares no code, header, table or helper with it.

Everything here is plain numpy in float64 (integers where the method is integer), written from
the definitions on the source pages:

* "Repacked QAT Gemma 4 26B-A4B serves on one TPU v6e at 1.9x FP8 throughput" (deniz.in),
  sections "A repack, not a re-quantization" (grid, group, scale trap, m-search, least-squares
  refine, verification) and "What changed in vLLM's TPU backend" (per-group scales, tile
  dequantised before the multiply, bf16 activations);
* "The Quantization Problem I Didn't Know I Had Until I Tried Running LLMs Locally"
  (adilsher.pro), section "Building the Missing Piece" (the repack steps);
* "What quantization really is" (janbancerewicz.github.io), section "How the ruler works"
  (symmetric scale-times-integer dequantisation).

Modules:
  bf16    bf16 <-> float64 (the storage type of activations and scales)
  q4      Q4_0 grid, packed-code layout, dequantisation, scale recovery (repack)
  linear  weight-only W4A16 dense linear
  moe     top-k routing and permutation, grouped expert GEMMs, GELU gate, combine

Where the pages leave a step open, the reading taken is stated in the function's docstring.
Pins that tie each function to something other than itself live in ``tests/test_oracle_*.py``.
The tanh-GELU gate is not on the pages (a reading: the tanh form of GELU); ``moe.gelu_tanh`` is
pinned to mathematical identities, to the erf form, and to PyTorch's tanh-approximate GELU, an
independent implementation of the same published approximation.
"""
