"""pagedattention_block_table_b200 -- PagedAttention hot path for B200 (sm_100a).

``binding``  ctypes face of libpagedattn.so (the CUDA kernels and their C ABI)
``runner``   device-side set-up of a paged batch and one serving step through the binding
``inputs``   seeded synthetic workloads (inputs only)
``build``    nvcc build of libpagedattn.so
"""
__all__ = ["binding", "runner", "inputs", "build"]
