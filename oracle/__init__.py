"""CPU oracle for the DSA forward path: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s ``cpu_baseline``
and ``--impl reference`` legs may import it. See ``oracle/dsa_oracle.py``.
"""
from .dsa_oracle import *  # noqa: F401,F403
from .dsa_oracle import __all__  # noqa: F401
