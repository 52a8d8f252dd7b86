"""Exact tiled attention with online softmax for B200 (sm_100a)."""
