"""NVFP4 attention forward with selective FP16 block pairs, for B200 (sm_100a).

The compute path is the C-ABI library ``libthrift_nvfp4.so`` built from
``csrc/``; ``ops`` is a thin ctypes binding over it.  Importing the package
does not load the library; the first call does, and fails loudly when the
library or a CUDA device is missing.
"""
