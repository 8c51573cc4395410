"""CPU oracle for the weight-informed activation-sparse linear layer.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` use it. It shares no code with the CUDA
library and does not import it.
"""

from .wina_oracle import *  # noqa: F401,F403
from .ds_oracle import *  # noqa: F401,F403
