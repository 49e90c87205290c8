"""Plain CPU oracle of the NVFP4 x Q8_0 dequantise-and-dot product.

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the CPU
legs of ``bench.py`` may import this package; the library never does.
"""
from .nvq_oracle import *  # noqa: F401,F403
from .nvq_oracle import __all__  # noqa: F401
