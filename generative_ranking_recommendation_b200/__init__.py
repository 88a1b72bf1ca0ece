"""GenRank hot path on B200 (sm_100a): action-oriented input assembly and
candidate-masked ALiBi attention, forward and backward, behind the C ABI of
libgenrank.so (include/genrank.h).

``genrank`` is the ctypes binding (same names as the C entry points);
``model`` wires it into the scoring and training steps of the workloads.
"""

__all__ = ["genrank", "model"]
