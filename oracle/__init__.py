"""fp64 CPU oracle for exact scaled-dot-product attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import anything here.  The product (the CUDA library and its
Python binding) never imports, calls or links this package, and this package
never imports the product: the two share no code.  Inputs come from the
neutral ``workloads`` module, which holds no attention arithmetic.

Modules
  reference   plain numpy fp64 forward/backward (explicit P, two-pass softmax)
  brute       pure-Python loops for tiny shapes (a second, independent pin)
  exp2_cubic  Cody-Waite range reduction + minimax cubic model of 2^x

Pins (tests/test_oracle.py) tie each function to facts the pages or the
mathematics fix: brute force, closed forms, invariants, finite differences,
library special cases and the minimax error bound.
"""
