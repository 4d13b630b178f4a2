"""B200-native beam-decode hot path of generative recommendation (xGR's
xAttention / xBeam), behind the C ABI of libxgr.so.

``xgr`` is the ctypes binding (same names as include/xgr.h); ``build`` compiles
the CUDA library in-tree for sm_100a; ``session`` wraps one context and its
workspace for convenience.
"""
