"""Oracle package: the plain fp64 CPU model that the CUDA path is checked against.

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()`` and
by the benchmark's CPU-baseline leg, never by the library itself.
"""
from .gpt_oracle import *  # noqa: F401,F403
from .gpt_oracle import Config  # noqa: F401
from .presets import PRESETS, preset  # noqa: F401
from . import optim_oracle as optim  # noqa: F401,E402
from . import fp8_oracle as fp8  # noqa: F401,E402
