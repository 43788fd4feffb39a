"""libmoedec: routed mixture-of-experts decode layer for B200 (sm_100a).

Submodules:
  moedec  -- ctypes binding of the C ABI (loads libmoedec.so; raises if absent)
  synth   -- seeded synthetic inputs shaped like the pages' workloads
  build   -- nvcc build of libmoedec.so in-tree
The binding is imported on first use so that `synth` and `build` work on a
machine where the library has not been built yet.
"""

__all__ = ["moedec", "synth", "build"]
