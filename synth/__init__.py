"""Seeded synthetic inputs for the sparse decode step (random draws and cache layout only)."""
from .inputs import (  # noqa: F401
    PAGE_SIZE,
    CONFIGS,
    DecodeProblem,
    make_problem,
    make_config,
    stream_seed,
)
