"""CPU oracle (fp64) for indexed sparse attention: test infrastructure only.

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline may import this package. The CUDA path never imports it.
"""
from .lsa_oracle import *  # noqa: F401,F403
from .lsa_oracle import __all__  # noqa: F401
