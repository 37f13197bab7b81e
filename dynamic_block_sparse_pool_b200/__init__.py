"""Dynamic block-sparse self-attention for video DiTs on B200 (sm_100a).

Pipeline per (batch, head): mean-pooled block scores with a row softmax,
per-row Top-p block selection (optionally restricted to a candidate set),
exact block-sparse attention over the selected blocks, and the exact softmax
mass of every selected block.  All arithmetic runs in ``libdsa.so``; the
Python layer only marshals arguments (see ``ops``).  The library is loaded
on the first call, and a call fails loudly if it has not been built.
"""
from . import ops, synth  # noqa: F401
from ._lib import DSAError  # noqa: F401
from .ops import (HilbertOrder, attn_bwd, attn_fwd, block_mass, device_status,  # noqa: F401
                  hilbert_order, mass_to_probs, permute_tokens, pool_score, pool_score_hier,
                  select_topp, sparse_attention)

__all__ = ["ops", "synth", "DSAError", "pool_score", "select_topp", "attn_fwd",
           "block_mass", "mass_to_probs", "sparse_attention", "device_status",
           "hilbert_order", "permute_tokens", "HilbertOrder", "pool_score_hier", "attn_bwd"]
