"""CPU oracle of the 4-bit weight-quantised linear layer.

TEST INFRASTRUCTURE ONLY: tests, the smoke check and the CPU legs of the
benchmark import it; the library never does. See ``wq_oracle`` for what it
computes and which page each step follows.
"""
from .wq_oracle import *  # noqa: F401,F403
from . import wq_oracle  # noqa: F401
