"""B200 (sm_100a) fused scaled-dot-product attention forward."""
