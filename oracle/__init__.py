"""CPU oracle for the DeltaKV hot path (test infrastructure; never imported by the product path)."""
from .deltakv_oracle import *  # noqa: F401,F403
from . import deltakv_oracle as core  # noqa: F401
