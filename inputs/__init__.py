"""Seeded synthetic input generators (no arithmetic of the method lives here)."""
from .synthetic import *  # noqa: F401,F403
from .synthetic import memory_sweep_input  # noqa: F401
