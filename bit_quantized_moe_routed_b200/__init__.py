"""B200-native routed-expert MoE FFN with MXFP4 / VQ13(+R8) compressed experts.

The compute lives in ``libmoeq.so`` (C ABI, ``include/moeq.h``); the
``moeq`` submodule is its ctypes binding.  Importing the binding fails when
the library has not been built: there is no other implementation.
"""

__all__ = ["moeq", "build"]
