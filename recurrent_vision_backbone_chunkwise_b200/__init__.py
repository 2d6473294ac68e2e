"""B200-native chunkwise key-gated linear attention (GTR's token mixer).

The compute lives in ``libgtr_gla.so`` (hand-written CUDA for sm_100a behind a
C ABI, declared in ``include/gtr_gla.h``); :mod:`.gla` is a thin ctypes
binding over it.  Nothing here falls back to a CPU implementation: if the
library is missing the binding raises.

Importing the package does not load the library; ``from
recurrent_vision_backbone_chunkwise_b200 import gla`` does.
"""
