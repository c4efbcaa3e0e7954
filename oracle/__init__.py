"""CPU oracle for the Veda tile-skip sparse-attention path.

TEST INFRASTRUCTURE ONLY. This package is a plain, slow, obviously correct restatement of what the
method computes, written from its published definition (the page ``veda_core.py`` of the
ComfyUI-FunPack node pack: sections "budgets", "tiles", "predictor", "selection", "one layer").
Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference`` legs of
``bench.py`` may import it. The product path (``learned_block_sparse_tile_b200``) never imports it and
shares no code with it; the two meet only through the seeded generators in ``veda_synth``.

Precision: integers exactly; budgets in IEEE double in the page's operation order; pooling, logits
and attention in float64 (tighter than the page's fp32), compared to the CUDA path with tolerances.

Every function is pinned by a ``-m "not gpu"`` test in ``tests/test_oracle_pins.py`` except where its
docstring says "parity unpinned".
"""
from .veda import *  # noqa: F401,F403
