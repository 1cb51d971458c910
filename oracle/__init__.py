"""CPU oracle (test infrastructure only; see nvfp4_oracle's header for who may use it)."""
from . import nvfp4_oracle  # noqa: F401
