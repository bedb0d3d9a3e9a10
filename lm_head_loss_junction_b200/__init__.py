"""Matryoshka LM-suite junction and multi-exit LM-head loss on B200 (sm_100a)."""
