"""Gecko sliding chunk attention + adaptive working memory forward for B200.

The compute path is the C-ABI library ``libgecko.so`` (hand-written sm_100a
CUDA) loaded by :mod:`long_context_sequence_sca_b200.lib`.  Import that module
explicitly; this package init stays free of side effects so the input
generator can be imported without the native library.
"""
