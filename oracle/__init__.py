"""CPU oracle for the AWQ hot path -- test infrastructure only (see ``awq_oracle``).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline leg import this
package. It shares no code with the CUDA library and never imports it.
"""
from .awq_oracle import *  # noqa: F401,F403
from .awq_oracle import __all__  # noqa: F401
