"""CPU oracle for layer-wise 4-bit post-training weight quantization (GPTQ + RTN).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
link this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code with the CUDA path (``post_weight_quantization_27_b200``).

Every function here is a plain, slow, obviously-correct restatement of what
the pages on this method define; see ``oracle/gq_oracle.py`` for the
citations and the readings taken where the pages are silent or garbled.
"""
from .gq_oracle import *  # noqa: F401,F403
