"""Block-scaled FP8 linear for B200 (sm_100a): Python binding of liblnq.so (placeholder)."""
