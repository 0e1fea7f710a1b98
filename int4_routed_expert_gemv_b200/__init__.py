"""Routed int4 MoE layer for B200 (sm_100a): router top-k, batch union, gs64 int4 SwiGLU
experts with routing-weighted combine, as a C-ABI CUDA library with a thin binding."""
