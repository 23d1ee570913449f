"""B200-native (sm_100a) Whisper-style audio encoder tower.

The compute lives in libenc_b200.so (hand-written CUDA behind the C ABI of
include/enc.h); this package only builds it and binds it with ctypes.
"""
from .binding import (Cache, Encoder, EncError, Frontend, clip_flops, encoder_config, load_library,  # noqa: F401
                      shard_plan, status_string)

__all__ = ["Cache", "Encoder", "EncError", "Frontend", "clip_flops", "encoder_config", "load_library", "shard_plan",
           "status_string"]
