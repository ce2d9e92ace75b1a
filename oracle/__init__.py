"""fp64 CPU oracle of the indexer step: test infrastructure, never used by the library."""
from . import lsa_oracle  # noqa: F401
