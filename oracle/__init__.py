"""fp64 CPU checker of the VSA forward pass -- TEST INFRASTRUCTURE ONLY.

Only tests/, the smoke check in __graft_entry__.py and the CPU-baseline leg
of bench.py may import this package. The CUDA library and its Python binding
never import it; the two implementations share no code.
"""
from .vsa_oracle import *  # noqa: F401,F403
from .vsa_oracle import __all__  # noqa: F401
