"""fp64 CPU oracle for the adaptive block-sparse attention path.

Test infrastructure only: imported by the tests, by the smoke check and by the
benchmark's CPU-baseline legs, never by the library.
"""
from .fvattn_oracle import *  # noqa: F401,F403
