"""Trie-constrained wide beam-search decode step, B200 (sm_100a) CUDA behind a C ABI."""
