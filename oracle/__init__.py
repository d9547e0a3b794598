"""CPU oracle (test infrastructure only; see lcsa_oracle's header)."""
from . import lcsa_oracle  # noqa: F401
