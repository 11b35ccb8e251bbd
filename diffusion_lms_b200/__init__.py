"""Route-layer chunk-routing sparse attention (Prefilling-dLLM v2) for B200, sm_100a.

The compute path is the CUDA library `librdl.so` behind a C ABI (include/rdl.h);
`diffusion_lms_b200.rdl` binds it.  Importing this package loads nothing; importing
`diffusion_lms_b200.rdl` loads the library and raises if it is missing.
"""
__all__ = ["workloads"]
