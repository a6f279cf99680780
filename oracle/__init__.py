"""CPU oracle for the Sparse-BitNet BitLinear forward.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The product path (``sparse_linear_layers_fwd_b200``) never imports, calls or
falls back to anything here.
"""

from .sbn_oracle import *  # noqa: F401,F403
from .sbn_oracle import __all__  # noqa: F401
