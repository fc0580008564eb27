"""CPU oracle for the NVFP4 W4A4 routed-expert MoE layer.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code, table or constant generator with the CUDA library.

The oracle is deliberately plain and slow: NumPy, IEEE fp32 element-wise
operations where the method fixes fp32 arithmetic, fp64 for every matmul and
for the layer's intermediate values.  Every function cites the passage of the
source pages it follows.  The pages print no formula and no quantised value for
NVFP4, so each step that they leave open follows a stated reading (the module
docstrings of ``oracle.nvfp4`` and ``oracle.moe`` list them).

Pins (what checks the oracle against something other than itself) live in
``tests/test_oracle_*.py``.  Functions with no external pin say
"parity unpinned" in their docstring.
"""
