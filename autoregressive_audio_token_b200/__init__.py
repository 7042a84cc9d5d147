"""B200-native (sm_100a) per-frame autoregressive decode of MiniMax Music 3's
Qwen3-style 8B "Global LLM" and its RVQ depth decoder.

The product is the C-ABI library libm3.so (include/m3.h); `m3` is its
ctypes binding under the same names.  There is no CPU fallback.
"""
from . import m3  # noqa: F401
from .m3 import M3Error  # noqa: F401
