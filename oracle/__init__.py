"""fp64 CPU oracle for sink attention -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py`` import it.
The CUDA path (``softmax_attn_sink_b200``) never does.  See ``oracle/ref.py``.
"""
from . import ref  # noqa: F401
