"""CPU oracle for grouped-query attention.

TEST INFRASTRUCTURE ONLY.  The product path (the C-ABI library and its Python
binding) never imports, links or runs anything in this package; only
``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` do.  It shares no code with the CUDA library.

Two independent restatements of the method:

* ``oracle.lab``  -- pure-Python brute force of the lab functions
  (TT Lab "キー・バリューヘッドだけ減らしてみる", steps 1-7), for tiny inputs;
* ``oracle.ref``  -- a C/OpenMP double-precision implementation of the plain
  definition for real shapes (forward, selected rows, decode, split decode
  merged by log-sum-exp), plus the bf16 tensor version of ``fold_kv``.
"""

from . import lab, ref  # noqa: F401
