"""bit_e8_lattice_b200 -- B200 kernels for 2-bit E8-lattice weight quantisation.

The compute lives in the CUDA library ``libe8q.so`` (C ABI, see
``include/e8q.h``); ``bit_e8_lattice_b200.e8q`` is the thin ctypes binding
with the same entry-point names.  ``synth`` draws the seeded inputs.
Importing this package loads nothing; the binding loads the library on
first use and raises if it is missing.
"""
__all__ = ["synth", "e8q"]
