"""fp64 CPU oracle for the MISA / MISA-dagger / HISA token indexer.

Test infrastructure only: the test suite, the smoke check and the benchmark's
CPU-baseline leg use it; the library never imports it.
"""
from .misa_oracle import *  # noqa: F401,F403
