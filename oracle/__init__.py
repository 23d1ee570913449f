"""CPU oracle of the audio encoder tower (test infrastructure only).

Imported by the tests, the smoke check and the benchmark's CPU-baseline leg;
never by the product library or its binding.
"""
from .encoder import *  # noqa: F401,F403
