"""Float64 CPU oracle for TurboQuant-style compressed-KV decode attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it. It shares
no code with the CUDA library (``decode_attention_seeded_b200``): the seeded
random tables, the Lloyd-Max codebooks, the rotation, the quantizer, the packed
page layout and the decode are all written out again here, slowly and plainly,
in float64 NumPy.

What it follows (pages are cited by title and section):

* "TurboQuant : 6x moins de cache, jusqu'a 8x plus rapide" (leviatan.io),
  sections "Principe de quantification sans calibration" and "Benchmarks de
  memoire": a linear transform of each K/V vector, no dataset-specific
  parameters, no per-block scale overhead.
* The korben-style llama.cpp-fork post (wis-web.com reader page), paragraphs on
  PolarQuant (Walsh-Hadamard rotation that makes the coordinate law known,
  then a radius plus a direction) and QJL (a 1-bit corrector that removes the
  residual inner-product bias).
* "To uger efter TurboQuant-papiret ..." (snilld.dk), section "Hvad papiret
  haevder": training-free and data-oblivious.

Where the pages leave a step open, the reading taken is stated in the
function's docstring. Modules:

``rng``       SplitMix64 stream, random sign vectors, fp16 Gaussian sketch S.
``hadamard``  natural-order fast Walsh-Hadamard transform and the rotation.
``codebook``  Lloyd-Max scalar codebooks (sphere marginal and Gaussian).
``quantize``  per-vector quantizer (norm, rotation, codes, QJL residual bits).
``layout``    byte layout of one 16-token page per KV head (pack / unpack).
``decode``    query transform, logit estimator, softmax, value sum, paged decode.

Parity status: every function is pinned by ``tests/test_oracle_*.py`` against
closed forms, textbook tables, published test vectors, brute force or
statistical identities; none is "parity unpinned".
"""

from . import rng, hadamard, codebook, quantize, layout, decode  # noqa: F401
