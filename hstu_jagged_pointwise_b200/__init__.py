"""Jagged HSTU pointwise attention for B200 (sm_100a).

The product is the C-ABI library ``libhstu_b200.so`` (``include/hstu.h``);
``hstu_jagged_pointwise_b200.ops`` is its torch-facing binding (``Layer``,
``MFalcon``, ``debug_indices``).  ``workloads`` draws seeded synthetic inputs.
Importing this package loads nothing; importing ``ops`` loads the library and
fails loudly if it has not been built.
"""
__version__ = "0.1.0"
