"""mao: matrix-aware optimizer steps (Muon, Muon+, SOAP, FOAM) on B200.

The compute lives in the C-ABI library ``libmao.so`` (hand-written sm_100a CUDA);
``matrix_aware_optimizers_02_b200.api`` is the thin Python binding over it.
``synth`` holds the seeded synthetic input generators.
"""

__all__ = ["api", "synth"]
