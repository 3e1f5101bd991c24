"""Test-infrastructure oracle (fp64, CPU).  Not part of the product path."""
from .moe_oracle import *  # noqa: F401,F403
