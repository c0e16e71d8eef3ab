"""fp64 CPU oracle (test infrastructure only; see mlstm_oracle's header)."""
from .mlstm_oracle import *  # noqa: F401,F403
from .mlstm_oracle import SIG, EXP  # noqa: F401
