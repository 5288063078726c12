"""KV-COBRA transform-coded low-bit KV cache for B200 (sm_100a).

The compute path lives in the C-ABI shared library ``libkvtc.so`` (CUDA kernels for
sm_100a plus a C++ host side for calibration).  ``bit_quantization_head_b200.kvtc``
is a thin ctypes binding with the same entry-point names; it only marshals
arguments.  Importing this package does not load the library; ``kvtc.lib()`` does,
and raises if it is missing.  There is no CPU fallback.
"""

__all__ = ["kvtc", "synth"]
