"""CPU oracle of the TTT-E2E inner loop: test infrastructure, never on the product path."""
from .ttt_oracle import Oracle  # noqa: F401
