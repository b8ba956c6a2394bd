"""InfLLM v2 sparse attention for NVIDIA B200 (sm_100a).

The work happens in ``libinfllmv2.so`` (hand-written CUDA behind a C ABI, declared in
``include/infllmv2.h``).  ``trainable_block_sparse_v2_b200.binding`` is a thin ctypes layer with the
same function names; it loads the library on first use and raises if it is missing -- there is no
CPU fallback.  ``workloads`` generates the seeded synthetic inputs.
"""
__all__ = ["binding", "workloads"]
