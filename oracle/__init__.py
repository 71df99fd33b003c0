"""Float64 CPU oracle for paged sparse-KV attention.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference leg of ``bench.py`` may import or run anything here.
The library in ``paged_sparse_kv_sa_b200`` never imports it, and the oracle
imports nothing from the library: the two share no code.  Inputs reach the
oracle as plain arrays (bf16 bit patterns as ``uint16``, tables as ``int32``).

Every function follows the plain definition of what the method computes and
cites the passage it restates.  Pins that tie the oracle to something other
than itself live in ``tests/test_oracle_pins.py``.
"""
from .sa_oracle import *  # noqa: F401,F403
