"""CPU oracle of the tile-binned Gaussian splatting rasterizer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library and its Python binding never import it, and it never imports them.
"""
from .oracle import *  # noqa: F401,F403
from . import train  # noqa: F401
from . import features  # noqa: F401,E402
