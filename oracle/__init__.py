"""Oracle for the KV-COBRA transform-coded KV cache.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, fp64 (numpy) restatement
of what the KV-COBRA project page ("KV-COBRA: KV Cache Compression via Co-Optimized
Bit-Rank Allocation") says the method computes.  It exists to check the CUDA path.
Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its cpu_baseline leg
and its ``--impl reference`` arm) may import it.  The product package
``bit_quantization_head_b200`` never imports it, and it never imports the product:
the two share no code.  Seeded inputs come from ``bit_quantization_head_b200.synth``,
which holds no arithmetic of the method; callers pass the arrays in.

Modules:
  calibration  per-head eigenbasis, attention-KL weights, D(r,b), C1, C2,
               random-sign Walsh-Hadamard folding, Gaussian quantizer step
  codec        canonical fp32 projection, b-bit uniform quantizer, page layout
  attention    decode attention over the compressed cache, in the original d-space

Parity status of each function (what pins it) is listed in its docstring; functions
without an independent pin say "parity unpinned".
"""

from . import calibration, codec, attention  # noqa: F401
