"""CPU oracle for the Attamba layer's forward hot path.  TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, float64 (numpy) restatement of what the Attamba
attention layer computes, written from the method's published description
("Attamba: Attending To Multi-Token States", arXiv 2411.17685, as summarised on
the codewithpapers.app abstract page, the rohan-paul.com summary and the
pith.science review).  It exists only so that the CUDA path can be checked
against something that a reader can verify by eye.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it; the product path never does, and it shares
no code, table or helper with the CUDA library.

Modules
-------
chunks     chunk boundaries: uniform size P, cyclic offset, variable lengths
ssm        the selective state-space scan (KV-SSM) with reset at chunk starts
mask       M_train / M_test / leading-token masks, dense from the definition,
           and the canonical compact key index derived from the same definition
attention  dense masked softmax attention (whole rows and sampled rows)
decode     one-token-at-a-time decode over the boundary-state cache
projection the layer's linear projections (kept W_Q, W_O; the SSMs' Delta, B, C)
scalar     literal scalar loops for tiny shapes (brute-force cross-check)

Every function states which passage it follows.  Where the pages are silent the
reading taken is stated in the docstring; the full list is in the repository's
design notes.  Every function is pinned by ``tests/test_oracle_*.py`` against
closed forms, invariants, brute force and the page's own worked count.
"""

from . import chunks, ssm, mask, attention, decode, projection, scalar  # noqa: F401
