"""CPU oracle (test infrastructure only): see moe_null_oracle.py."""
from .moe_null_oracle import *  # noqa: F401,F403
from .moe_null_oracle import __all__  # noqa: F401
