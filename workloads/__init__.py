"""Seeded synthetic inputs shared by the tests, the smoke check and the bench."""
from .synth import (CONFIG_NAMES, Workload, make_decode, make_local_decode, make_prefill,  # noqa: F401
                    make_workload, random_scores)
from .attention import MlaBatch, make_mla, mla_cache_rows  # noqa: F401
