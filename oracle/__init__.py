"""CPU oracle for the LLSA hot path (test infrastructure; see llsa_oracle.py)."""
from . import llsa_oracle  # noqa: F401
