"""Block-quantised weight GEMV for B200 (sm_100a): the LLM decode hot path.

The compute lives in the CUDA shared library ``libbq.so`` (C ABI declared in
``include/bq.h``); :mod:`quantised_weight_gemv_b200.bq` is a thin ctypes
binding with the same names.  :mod:`quantised_weight_gemv_b200.synth` draws the
seeded synthetic inputs.  Importing the package loads nothing.
"""
