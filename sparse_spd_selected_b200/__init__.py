"""libselinv: batched block selected inverse of sparse SPD matrices on B200.

The compute path is the C-ABI shared library ``libselinv.so`` (hand-written
sm_100a CUDA kernels) in this package directory; ``selinv`` is its thin
ctypes binding.  Importing the package does not load the library; the first
call into ``selinv`` does, and fails loudly if it has not been built.
"""
__all__ = ["selinv", "inputs"]
