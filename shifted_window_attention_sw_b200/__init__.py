"""B200-native 3D (shifted-)window multi-head self-attention (Video Swin W-MSA / SW-MSA).

The layer runs in ``libvswin.so`` (hand-written CUDA for sm_100a, C ABI in
``include/vswin.h``); ``vswin`` is its ctypes binding.
"""

from . import vswin  # noqa: F401
from .vswin import (  # noqa: F401
    VswinError,
    clamp_window,
    index_maps,
    wmsa_forward,
    wmsa_forward_f32,
    wmsa_forward_host,
)
