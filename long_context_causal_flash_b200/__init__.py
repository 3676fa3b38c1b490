"""Exact causal grouped-query attention for B200 (sm_100a) behind a C ABI."""
