"""B200-native routed-expert MoE layer with decoupled top-k1 / top-k2
renormalisation (Eq. 2 of "Paper of the Week #3 -- Half the FLOPs Is Not Half
the Time", section "The Receipt").

Submodules:
  moe    -- ctypes binding of the C-ABI library libmoe.so (same call names);
  synth  -- seeded synthetic inputs;
  build  -- nvcc build of libmoe.so for sm_100a.

Importing the package loads nothing; ``moe`` loads libmoe.so on first use and
raises if it is missing.
"""
__all__ = ["moe", "synth", "build"]
