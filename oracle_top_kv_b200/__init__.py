"""HySparse / HySparse2 hot path on B200 (sm_100a): C-ABI library + thin Python binding."""
