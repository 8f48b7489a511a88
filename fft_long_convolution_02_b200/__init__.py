"""B200-native Hyena gated FFT long convolution.

The operator ([P4] "HyenaDNA operator walk-through" (adg.csdn.net), section
二.1; [P5] "Native Multi-Dimensional Subquadratic Operators via Input
Dependent Long Convolutions", 方法论) runs in the CUDA library
``libhyena_b200.so`` behind the C ABI of ``include/hyena.h``; ``binding``
marshals torch tensors into it.  ``inputs`` holds the seeded synthetic
workloads.  Importing the package does not load the CUDA library; the first
binding call does, and raises if it has not been built.
"""
from .binding import (HyenaError, hyena_filter_spectrum, hyena_gated_fftconv,  # noqa: F401
                      hyena_gated_fftconv_workspace_bytes, hyena_gated_fftconv_workspace_min_bytes,
                      hyena_shortconv, hyena_spectrum_bytes, hyena_spectrum_check, hyena_version, load)
