"""CPU oracle for partitioned attention-state reuse.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute anything in this package: only ``tests/``, ``__graft_entry__.smoke()``
and the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.
It shares no code with the CUDA library and imports nothing from it.

Every function is a plain float64 numpy restatement of what the two source
pages define; see ``attention_state.py`` for the per-function citations and
for which readings of the pages it takes where they are silent.
"""

from .attention_state import *  # noqa: F401,F403
