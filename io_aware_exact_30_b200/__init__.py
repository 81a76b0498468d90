"""B200-native exact attention: tiled forward with online softmax and a
recompute backward, behind the C-ABI library ``libattn.so``.

The Python layer is argument marshalling only; see :mod:`.attn`.
"""

__all__ = ["attn", "synth"]
