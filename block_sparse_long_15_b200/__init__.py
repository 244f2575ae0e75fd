"""QSA (Qwen Sparse Attention) hot path for NVIDIA B200.

Submodules:
  qsa        -- ctypes binding of the C ABI in include/qsa.h (loads libqsa.so)
  runner     -- device buffers + calls for prefill and decode through qsa_forward
  workloads  -- seeded synthetic inputs
  build      -- nvcc build of libqsa.so for sm_100a
The binding is imported lazily so that building and input generation work on
machines without the compiled library.
"""
__all__ = ["qsa", "runner", "workloads", "build"]
