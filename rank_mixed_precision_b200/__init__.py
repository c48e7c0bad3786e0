"""STAR-KV latent-cache attention for B200 (sm_100a): C ABI + thin torch binding.

The compute lives in ``libstarkv.so`` (CUDA kernels for sm_100a); ``starkv``
marshals torch tensors into its C entry points.
"""
from . import starkv  # noqa: F401
from .starkv import LatentCache, StarKV, StarKVError, make_config  # noqa: F401
