"""fp64 CPU oracle of the generalized delta-rule recurrence.

TEST INFRASTRUCTURE: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (``matrix_memory_rnn_b200``) never does.
"""
from .oracle import (FORMS, backward, build, decode_step, forward, library_path, load_library,
                     max_threads, mlstm_forward, muir_forward)  # noqa: F401
