"""Float64 CPU oracle for reduced-KV softmax decode attention.

Test infrastructure only: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.
"""
from .oracle import *  # noqa: F401,F403
from . import oracle as impl  # noqa: F401
