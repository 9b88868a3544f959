"""B200-native (sm_100a) fine-grained MoE expert layer: a C-ABI CUDA library
(libmoe.so, include/moe.h) and its thin ctypes binding (`moe`)."""
