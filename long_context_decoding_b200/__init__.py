"""long_context_decoding_b200 -- combined sparse decode attention on B200.

The CUDA library (``libcsa.so``, C ABI declared in ``include/csa.h``) is
loaded lazily by :mod:`long_context_decoding_b200.csa`; importing the package
itself needs no GPU.  :mod:`long_context_decoding_b200.workloads` holds the
seeded synthetic inputs.
"""
__all__ = ["csa", "workloads"]
__version__ = "0.1.0"
