"""Lighthouse Attention layer for B200 (sm_100a): C-ABI library and its Python binding."""
