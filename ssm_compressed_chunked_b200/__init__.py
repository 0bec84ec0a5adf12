"""Attamba layer forward hot path on B200 (sm_100a).

The compute lives in ``libattamba.so`` (hand-written CUDA behind a C ABI, see
``include/attamba.h``); ``ssm_compressed_chunked_b200.attamba`` is the thin
ctypes binding that passes torch tensors' device pointers and the current
stream into it.  ``workloads`` draws the seeded synthetic inputs.

Importing this package loads nothing; the binding loads the library on first
use and raises if it is missing.
"""
