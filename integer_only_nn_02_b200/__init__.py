"""B200-native integer-only (C,e) training kernels.

Every tensor is a pair (C,e): INT8 mantissas with a power-of-two exponent per group
("Memory-Efficient Integer-Only Training of Deep Neural Networks", Abstract and
Figure 1).  The compute path is the C-ABI library ``libict.so`` (sm_100a kernels);
``integer_only_nn_02_b200.ict`` is its thin Python binding and
``integer_only_nn_02_b200.workloads`` holds the seeded synthetic inputs.

Importing the package itself loads nothing; importing ``.ict`` loads ``libict.so``
and raises if it is missing.
"""

__all__ = ["ict", "workloads"]
