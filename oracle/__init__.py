"""fp64 CPU oracle of the ViT encoder hot path -- TEST INFRASTRUCTURE.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA
library.  See ``oracle/vit_ref.py`` for the definitions and the readings of
the pages they follow.
"""
from .vit_ref import *  # noqa: F401,F403
from . import vit_ref  # noqa: F401
