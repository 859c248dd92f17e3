"""fp64 CPU oracle for the MISA / MISA-dagger / HISA token indexer and the
sparse attention over the tokens it selects.

Test infrastructure only: the test suite, the smoke check and the benchmark's
CPU-baseline leg use it; the library never imports it.
"""
from .misa_oracle import *  # noqa: F401,F403
from .attention_oracle import *  # noqa: F401,F403
