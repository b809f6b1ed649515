"""fp64 CPU oracle for MoBA causal prefill (test infrastructure only; see moba_oracle)."""
from .moba_oracle import *  # noqa: F401,F403
from .moba_oracle import __all__  # noqa: F401
