"""StreamBP streamed exact backward for B200 (sm_100a).

The compute lives in ``libsbp.so`` (hand-written CUDA behind a C ABI); ``sbp`` is its ctypes
binding.  Importing the package loads nothing: ``sbp.load()`` opens the library.
"""
__all__ = ["synth", "sbp"]
