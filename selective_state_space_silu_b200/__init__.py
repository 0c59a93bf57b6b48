"""B200-native fused Mamba-1 selective-SSM mixer core.

``mixer`` holds the Python binding of the C-ABI library ``libmamba_mixer.so``
(causal conv1d + SiLU, softplus, selective scan, gate, and the single-token decode
step, all in hand-written sm_100a CUDA kernels).  ``inputs`` draws seeded synthetic
inputs.  Importing the package loads nothing; the library is loaded on first use and
its absence is an error, never a fallback.
"""

__version__ = "0.1.0"
