"""CPU oracle for the S + U Vᵀ compressed linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``sparse_rank_linear_03_b200``) never imports it,
and this package imports nothing from the product.

Every function here is plain, slow, obviously-correct NumPy in float64 (the
pages fix no precision).  See ``oracle/hss.py`` for the citations and for which
functions are pinned by which tests.
"""
from .hss import *  # noqa: F401,F403
