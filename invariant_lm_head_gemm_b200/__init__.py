"""Bitwise batch-invariant linear-logp (LM head -> logp, entropy, lse and
their backward) for B200 (sm_100a)."""
