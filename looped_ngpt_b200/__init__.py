"""B200-native elastic-depth forward pass of the Dory1.0-4B looped nGPT.

The compute path is ``libdory.so`` (hand-written sm_100a CUDA behind the C
ABI in ``include/dory.h``); this package only marshals arguments and uses
PyTorch for device memory and streams.
"""
from ._lib import load, LIB_PATH, DoryError, KV_MODES
from .model import DoryModel, KVCache, to_device

__all__ = ["load", "LIB_PATH", "DoryError", "KV_MODES", "DoryModel", "KVCache",
           "to_device"]
