"""CPU oracle for the LoopVQ hot path (test infrastructure only).

This package is a plain, slow, fp64 NumPy restatement of what the LoopVQ
pages define: loop-axis sub-vector formation, brute-force nearest-codeword
encoding, per-loop-step dequantization through the codebook slice, and naive
softmax decode attention over a bf16 sink/recent window plus the quantized
body.  It shares no code with the CUDA library and imports nothing from it.

Only the test-suite, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it.  The product path
(the C-ABI library and its Python binding) never calls it.
"""
from .loopvq_oracle import *  # noqa: F401,F403
