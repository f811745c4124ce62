"""CPU oracle for the compressed-KV sparse decode-attention path.

This package is test infrastructure. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it. The product path
(the CUDA library and its Python binding) never imports, calls or links anything here.
"""

from .ckv_oracle import *  # noqa: F401,F403
