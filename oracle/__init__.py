"""CPU oracle for VideoMLA latent-KV attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path never calls it, and it shares no code with the CUDA library.
"""
from .mla_oracle import *  # noqa: F401,F403
