"""Exact IO-aware attention for B200 (sm_100a): C-ABI library and its Python binding."""
