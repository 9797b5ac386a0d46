"""sigattn: sigmoid attention over padded variable-length batches on B200 (sm_100a).

The compute lives in ``libsigattn.so`` (hand-written CUDA kernels behind a C ABI,
declared in ``include/sigattn.h``); ``binding`` is a thin ctypes layer over it.
"""
