"""B200-native (sm_100a) SVDQuant W4A4 linear layer.

The compute lives in libsvdq.so (C ABI: include/svdq.h), built in-tree by
`python -m bit_diffusion_transformer_svdq_b200.build`.  `svdq` is the thin
ctypes binding with the same function names.
"""
