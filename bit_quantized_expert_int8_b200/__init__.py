"""B200-native MoE decode hot path: int8 router, 4-bit affine group-quantised
expert FFNs, weighted combine and a per-layer LFU expert cache, as hand-written
sm_100a CUDA kernels behind the C-ABI library ``libmoeq4.so``."""
