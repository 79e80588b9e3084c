"""Plain CPU fp64 oracle for ring / striped / Ulysses attention.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library and
its Python binding) imports, links or calls this package; only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline legs of ``bench.py`` do.  It
shares no code with the CUDA path: no kernels, headers, helpers, tables or
pre/post-processing.  The only thing both sides consume is the seeded input
generator, which lives in a module of its own and holds none of the method's
arithmetic.

Everything here is written to be checked by eye against the pages it cites:
- "Mosaic: Sharding Attention Across GPUs When Your Sequence Doesn't Fit"
  (dev.to, P. Sateesh), sections "The Problem", "How Ring Attention Works",
  "The Implementation", "Beyond 1D: Mesh2D Attention";
- "ringmaster" (PyPI page of axolotl-ringmaster 0.2.0), sections "Why",
  "Status", "Layout";
- "Ring Attention & Friends" (slide deck), slides "Vanilla Transformer",
  "Flash Attention - Tiling with the Softmax Rescaling Trick",
  "Striped Attention".

All floating point is numpy float64.  The full score row of every query is
materialised (queries are processed in row blocks so that a 131k-token
sequence does not need a 137 GB matrix); there is no online softmax and no
tiling of the key axis anywhere in this package.

Modules:
- ``attention``  exact attention forward / backward on one (Q, KV) pair,
                 optionally packed or right-padded (segment ids)
- ``merge``      LSE merge of partial (O, LSE) results
- ``layouts``    contiguous / zigzag / striped global-position maps, permutes
- ``ring``       the ring over P ranks (forward and backward)
- ``repack``     Ulysses sequence<->head repack as explicit index loops
- ``multiaxis``  row-axis / feature-axis routing of a tabular tensor
- ``usp``        Ulysses x ring composition (USP) and its degree selection
- ``mesh2d``     Mesh2D: tiles of a (query chunk x key chunk) grid, merged

Parity status: every function above is pinned by ``tests/test_oracle_*.py``
(closed forms, brute force, invariants, finite differences, a library
cross-check); none is "parity unpinned".
"""

from . import attention, layouts, merge, mesh2d, multiaxis, repack, ring, usp  # noqa: F401
