"""FP64 CPU oracle of the W4A16 weight-only INT4 linear layer.

TEST INFRASTRUCTURE ONLY: the test-suite, the smoke check and the benchmark's CPU-baseline leg
are the only users. The product library never imports it, and it never imports the product.
"""
from .oracle import *  # noqa: F401,F403
