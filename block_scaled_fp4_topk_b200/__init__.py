"""B200-native (sm_100a) block-scaled FP4 routed-expert MoE FFN.

``ds4g``  -- thin binding of the C ABI in include/ds4g.h (libds4g.so)
``layer`` -- one MoE layer as the sequence of library calls
"""
from . import build  # noqa: F401
