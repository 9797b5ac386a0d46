"""Float64 CPU oracle for padded variable-length sigmoid / softmax / softmax_1 attention.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it.  It shares no code with the CUDA library (no kernels,
headers, helpers or tables); both sides take their inputs from
``padded_variable_length_b200.workloads``, which holds none of the method's
arithmetic.

Modules
  attention  vectorised float64 forward and analytic backward (the definition
             written out, row-chunked so no N x N matrix is ever held)
  brute      pure-Python loops for tiny shapes (a second, independent spelling)
  tiles      the 128 x 128 tile list (CSR / CSC / kinds / partial bitmasks) by
             brute-force any/all over each block

Pinning: every function here is checked in ``tests/test_oracle_pins.py`` against
closed forms, brute force, finite differences and invariants derived from the
pages ("Better Models, Faster Training: Sigmoid Attention for single-cell
Foundation Models"; "Binary Block Masking"; the softmax_1 / QuietAttention
page; the FlashAttention article).  No function is "parity unpinned".
"""
