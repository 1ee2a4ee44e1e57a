"""B200-native decode attention over a prunable 2-bit KV cache (Dual-QK).

Modules:
  kvq        -- Python binding of the C ABI in include/kvq.h (libkvq.so)
  workloads  -- seeded synthetic inputs shaped like the Dual-QK workloads
  build      -- nvcc build of libkvq.so for sm_100a
"""
__all__ = ["kvq", "workloads", "build"]
