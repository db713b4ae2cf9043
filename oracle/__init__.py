"""CPU oracle for the 4-bit Shampoo preconditioner step.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.
"""
from .shampoo4_oracle import *  # noqa: F401,F403
