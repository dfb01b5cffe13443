"""CPU oracle for SharQ's sparse-dense FP4 linear layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s ``cpu_baseline`` / ``--impl reference`` legs may import or run
anything here. The CUDA library (``fp4_activation_sparse_b200``) never imports
it and shares no code, table or constant generator with it.

Modules:
  formats -- E2M1 / E4M3 / E8M0 codes (tables from the bit fields; RNE encoders)
  sharq   -- RMSNorm, N:M mask, NVFP4/MXFP4 block quantizers, the preparation
             operator, the weight payload with two scale views, float64 GEMMs

Pins (the ``-m "not gpu"`` tests) tie each function to something other than
itself: library codecs (torch float8, ml_dtypes float4), brute force over all
subsets or all codes, closed forms and invariants, and hand-worked fixtures
under ``tests/golden``. The one inequality-only check is the method sanity
test (SharQ's output error below dense NVFP4's); it pins no value.
"""
from . import formats, sharq  # noqa: F401
