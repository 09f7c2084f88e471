"""Block Transformer global-to-local inference on B200 (sm_100a).

The compute path is the native library built from ``csrc/`` (CUDA kernels
behind the C-ABI of ``include/bt.h``); ``native`` is its ctypes binding and
``costmodel`` the bytes/FLOPs model used for rooflines. Importing this
package does not load the library; ``native.lib()`` does, and raises if it
has not been built.
"""
__all__ = ["native", "costmodel", "build"]
