"""B200-native fused Mamba-1 selective-SSM mixer core.

``mixer`` holds the Python binding of the C-ABI library ``libmamba_mixer.so``
(causal conv1d + SiLU, softplus, selective scan, gate, the single-token decode step and
the backward, all in hand-written sm_100a CUDA kernels); ``ssd`` binds the same library's
Mamba2 scan (chunked, on the tensor cores).  ``inputs`` draws seeded synthetic inputs.  Importing the package loads nothing; the library is loaded on first use and
its absence is an error, never a fallback.
"""

__version__ = "0.1.0"
