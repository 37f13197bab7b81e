"""Dynamic block-sparse self-attention for video DiTs on B200 (sm_100a).

Pipeline per (batch, head): mean-pooled block scores with a row softmax,
per-row Top-p block selection (optionally restricted to a candidate set),
exact block-sparse attention over the selected blocks, and the exact softmax
mass of every selected block.  All arithmetic runs in ``libdsa.so``; this
package only marshals arguments to it.
"""
__all__ = ["synth"]
