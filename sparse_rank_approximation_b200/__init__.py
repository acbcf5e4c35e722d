"""ELSAA sparse + low-rank attention for B200 (sm_100a).

The compute path is the C-ABI library ``libelsaa.so`` built from the CUDA
sources under ``csrc/``; ``binding`` marshals arguments to it.  Importing the
package does not load the library; ``binding.lib()`` does, and raises if the
library is missing (there is no CPU fallback).
"""
