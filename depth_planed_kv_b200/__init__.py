"""B200-native RIPE verify-attention over a depth-planed KV cache.

Submodules:
  ripe   -- ctypes binding of the C-ABI library ``libripe.so`` (loads the
            CUDA build; raises if it is missing)
  synth  -- seeded synthetic inputs and the workload shapes
"""
