"""CPU oracle for the BitNet b1.58 BitLinear forward pass.

TEST INFRASTRUCTURE ONLY.  This package is imported by the test suite, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py`` and by
nothing else.  The product (``ternary_weight_linear_04_b200``) never imports
it, and it never imports the product: the two share no code.

Two independent implementations live here:

* ``oracle.reference`` -- NumPy, written straight from the formulas, for
  small shapes (the pins in ``tests/test_oracle_pins.py`` run against it);
* ``oracle.native``    -- ctypes front end of ``bitlinear_oracle.c``, the
  same definitions as scalar C loops (optionally OpenMP over rows), fast
  enough for full-size spot checks and for the timed CPU baseline.

Pages are cited by title and section (tags defined in ``bitlinear_oracle.c``):
[Production], [Additive], [No-Multiply].
"""
