"""CPU fp64 oracle (test infrastructure, not the product path).

Only tests, the smoke check and the benchmark's CPU-baseline legs may use it.
"""
from .ref import allowed, attention_probs, backward, forward, row_dot  # noqa: F401
