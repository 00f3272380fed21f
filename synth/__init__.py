"""Seeded synthetic inputs shared by the oracle tests and the CUDA path (no method arithmetic)."""
from . import philox, configs  # noqa: F401
