"""CPU oracle (test infrastructure): see vlm_oracle.py. Never imported by the product path."""
from . import vlm_oracle  # noqa: F401
