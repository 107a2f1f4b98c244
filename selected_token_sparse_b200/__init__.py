"""Paged / selected-token sparse attention for B200 (sm_100a).

The compute path is the C-ABI library ``libspa.so`` built from ``csrc/``;
``spa`` is its thin ctypes binding.
"""
