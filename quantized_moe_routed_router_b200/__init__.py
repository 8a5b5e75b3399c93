"""B200-native routed MoE half (router GEMV, on-device top-k, grouped expert GEMVs, weighted combine).

The compute runs in the CUDA library ``libts_moe.so`` behind a C ABI
(``include/ts_moe.h``); ``binding`` marshals arguments to it through ctypes.
"""
