"""fp64 CPU oracle for MLA latent-KV decode.

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and ``bench.py``'s
CPU-baseline / reference legs may import it.  The library never does.
"""
from . import mla_oracle  # noqa: F401
