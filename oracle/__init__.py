"""fp64 CPU oracle of the SparsePR per-call sparse attention path.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline / reference leg, never by the product path.
"""
from . import sparsepr_oracle  # noqa: F401
