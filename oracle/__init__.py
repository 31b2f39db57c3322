"""Plain fp64 CPU oracle for the Wan full self-attention hot path.

TEST INFRASTRUCTURE ONLY: ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` are its only users.  The product path
(``video_dit_full_b200``) never imports, links or runs anything here, and
nothing here imports the product path; the two share only the seeded input
generator in ``synth``.

Parity pins: every function here is checked in ``tests/test_oracle*.py``
against brute force, closed forms, invariants and finite differences (see
those files).  The 8-bit recipe is simulated in two independent forms:
``quant8.attn_fwd_q8_sim`` (each block's V scale folded into P, one
accumulation) and ``quant8.attn_fwd_q8_blockwise`` (each block's 8-bit product
dequantised on its own and accumulated across blocks).  They are pinned to each
other (equal wherever no P code is subnormal), to the uniform-score closed form
and to the exact oracle's error budget; the 8-bit path's parity gate is the
unquantised ``attention.attn_fwd``.
"""
from .attention import attn_bwd, attn_fwd, softmax_matrix, widen  # noqa: F401
from . import quant8  # noqa: F401
