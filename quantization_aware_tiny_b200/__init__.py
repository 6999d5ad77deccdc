"""B200-native int6 quantization-aware linear, ReLU^2 MLP, recurrent-core
weight cache and export quantizer.

The compute path is the C-ABI CUDA library ``libqat_b200.so`` (sm_100a);
``quantization_aware_tiny_b200.qat`` is its thin ctypes binding.  Importing
this package loads nothing; the binding loads the library on first use and
raises if it is missing -- there is no CPU fallback.
"""
__all__ = ["qat", "synthetic"]
