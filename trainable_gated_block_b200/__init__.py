"""SAS gated block-sparse causal attention on B200 (sm_100a).

The compute path is the C-ABI library ``libsas.so`` (hand-written CUDA for
sm_100a); ``trainable_gated_block_b200.sas`` is a thin ctypes binding to it.
Importing this package loads nothing; the binding loads the library on first
use and raises if it is missing.
"""
