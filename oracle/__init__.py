"""CPU oracle (test infrastructure only; never imported by the product path)."""
from . import svdq_oracle  # noqa: F401
