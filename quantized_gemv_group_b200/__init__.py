"""quantized_gemv_group_b200 -- low-bit weight-only GEMV/GEMM for B200 (sm_100a).

The compute lives in the C-ABI library ``liblbq.so`` (CUDA kernels under
``csrc/``); ``lbq`` is its thin ctypes binding.  ``synth`` draws the seeded
synthetic inputs and ``workloads`` holds the shape and bit-schedule tables.
"""
__all__ = ["lbq", "synth", "workloads"]
