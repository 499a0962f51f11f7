"""The oracle: a plain, slow CPU statement of the BitLinear forward.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import anything here.  The product
(``ternary_weight_linear_token_b200``) never imports it and shares no code
with it; the only thing both sides use is the seeded input generator
(``synth``), which holds none of the method's arithmetic.

Two independent statements live here:

* ``ref`` -- ctypes wrapper of ``bitnet_ref.c`` (plain C99, fp64 gamma in a
  fixed order, int64 dot products written as the product sum).
* ``ref_np`` -- a numpy restatement that reaches the same numbers another
  way (the add/subtract form of the ternary product, numpy rounding done in
  fp64), used to cross-check the C oracle.

Parity status of each function is recorded in ``ref.PINS``.
"""
