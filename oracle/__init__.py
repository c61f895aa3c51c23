"""fp64 CPU oracle of the column-sparse cross-step delta method.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the CPU
legs of the bench, never by the library.
"""
from .chipmunk_oracle import *  # noqa: F401,F403
