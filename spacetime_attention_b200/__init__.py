"""B200-native spacetime attention: 3D RoPE, 3D full attention and Skiparse attention.

The compute lives in ``libosp.so`` (hand-written CUDA for sm_100a behind a C ABI declared in
``include/osp.h``); ``spacetime_attention_b200.ops`` is a thin ctypes binding over it.
"""
