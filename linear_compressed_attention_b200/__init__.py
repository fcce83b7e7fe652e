"""B200-native EDiT linear compressed attention (sm_100a CUDA behind a C ABI).

Importing the package loads nothing; ``binding`` loads the shared library on
first use and raises if it is missing.
"""
__all__ = ["inputs", "binding"]
