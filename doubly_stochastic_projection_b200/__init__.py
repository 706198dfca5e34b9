"""B200 (sm_100a) kernels for the mHC Birkhoff projection and 4-stream residual mix.

The compute lives in ``libmhc_b200.so`` (hand-written CUDA, C ABI declared in
``include/mhc_birkhoff.h``).  :mod:`.api` marshals torch tensors into it;
:mod:`.inputs` draws the seeded synthetic workloads.  Importing the package
does not load the CUDA library; the first call into :mod:`.api` does, and
fails loudly if it has not been built.
"""
__version__ = "0.1.0"
