"""Seeded synthetic inputs shared by the oracle and the CUDA path (generation only)."""
from . import rng, workloads  # noqa: F401
from .workloads import WORKLOADS, VOTE_WORKLOADS, ScoreWorkload, VoteWorkload  # noqa: F401
