"""B200-native Re-ttention: statistically reshaped static block-sparse attention.

The compute path is the C-ABI library ``librt_b200.so`` (hand-written sm_100a
CUDA kernels: calibration, reshaped sparse step, CSR block-index build).
``sparse_attention_diffusion_rt_b200.rt`` is the thin ctypes binding with the
same names as the C entry points; ``inputs`` draws seeded synthetic workloads.
Importing this package loads nothing; the binding loads the library on first
use and raises if it is missing.  There is no CPU fallback.
"""

__all__ = ["rt", "inputs"]
