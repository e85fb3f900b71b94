"""Seeded synthetic workloads shared by the tests, the bench and the oracle
callers. Holds random draws and storage layouts only."""
from .synth import *  # noqa: F401,F403
