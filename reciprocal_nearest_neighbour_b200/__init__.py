"""Reciprocal nearest-neighbour matching on B200 (sm_100a)."""
