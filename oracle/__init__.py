"""fp64 CPU oracle (test infrastructure only; see gla_oracle.py)."""

from .gla_oracle import gla_bruteforce_head, gla_forward, gla_head, relu, sigmoid

__all__ = ["gla_bruteforce_head", "gla_forward", "gla_head", "relu", "sigmoid"]
