"""B200-native I2_S ternary x int8 matmul (BitNet b1.58 projections).

The compute path is the CUDA library ``libbitnet_i2s.so`` (kernels for
sm_100a behind a C ABI declared in ``include/bitnet_i2s.h``).  ``i2s`` is the
thin ctypes binding with the same call names; ``inputs`` draws the seeded
synthetic workloads.  Importing this package loads nothing; importing ``i2s``
loads the library and raises if it is missing.
"""
__all__ = ["i2s", "inputs"]
