"""CPU oracle (test infrastructure; never imported by the product path)."""
from .ulysses_oracle import *  # noqa: F401,F403
