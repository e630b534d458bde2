"""B200-native Hilbert-ordered block routing and block-sparse attention (FVAttn hot path).

The compute path lives in ``libfva.so`` (hand-written sm_100a CUDA behind a C ABI).
``adaptive_block_sparse_hilbert_b200.fva`` is the thin ctypes binding; importing this
package does not load the library, so the seeded input generator
(``adaptive_block_sparse_hilbert_b200.synth``) stays importable on machines without it.
"""
__all__ = ["fva", "migrate", "pipeline", "synth"]
