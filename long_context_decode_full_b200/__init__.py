"""HySparse2 Hybrid-Block decode attention for B200 (sm_100a).

``long_context_decode_full_b200.hs2`` is the thin Python binding over the
C-ABI library ``libhs2.so`` (argument marshalling only; every step runs in
the CUDA kernels).  ``long_context_decode_full_b200.synth`` builds seeded
synthetic decode workloads.
"""
__all__ = ["hs2", "synth"]
