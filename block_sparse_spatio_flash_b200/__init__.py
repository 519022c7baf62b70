"""B200-native block-sparse spatio-temporal attention (forward) for video-diffusion heads.

The compute path lives in the CUDA library ``libsvgattn.so`` (sm_100a); ``svg`` is its thin
ctypes binding (argument marshalling only). ``synthetic`` holds the seeded workloads.
Importing the package itself loads nothing; ``from block_sparse_spatio_flash_b200 import svg``
loads the library and raises if it is missing.
"""
__all__ = ["svg", "synthetic"]
