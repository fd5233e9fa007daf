"""CPU fp64 oracle for the approximate-attention prefill layer.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by
the bench's CPU-baseline / reference arm.  The product path never uses it.
"""
from .spava_oracle import *  # noqa: F401,F403
from . import spava_oracle  # noqa: F401
