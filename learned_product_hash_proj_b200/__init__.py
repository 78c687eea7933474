"""B200-native (sm_100a) Monodratic mixer: learned product-hash routing and
exact selected-set attention, as a C-ABI CUDA library (``libmono.so``, header
``include/mono.h``) with a thin ctypes binding (:mod:`.mono`).

Submodules:
  mono   -- the binding (loads libmono.so; raises ImportError if it is missing)
  synth  -- seeded synthetic workloads (no method arithmetic)
  build  -- nvcc build of libmono.so for sm_100a
"""
__all__ = ["mono", "synth", "build"]
