"""CPU oracle for group-wise low-bit weight quantization.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this package.  The CUDA library never reaches it.

Two independent implementations of the same definitions:

* ``c_oracle``  -- ctypes binding of ``cq_oracle.c`` (plain C99, scalar loops, own
  fp16/bf16 converters written from IEEE-754), threaded over rows/groups for speed;
* ``np_oracle`` -- a vectorised NumPy twin for small inputs, using NumPy's own float16
  conversion and ``packbits`` as library primitives.

Both cite the pages they follow (see the module docstrings).
"""
