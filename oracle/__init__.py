"""FP64 CPU oracle for incoherence-processed LDLQ on one linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.
The CUDA library never calls it and shares no code with it.

Every function is a plain, slow restatement of what the pages define, in
float64 NumPy, written so it can be checked against the text by eye.  See
``oracle/quip_oracle.py`` for the citations and for which functions are
pinned by which tests.
"""
from .quip_oracle import *  # noqa: F401,F403
from .quip_oracle import __all__  # noqa: F401
