"""CPU oracle (test infrastructure only): see ``oracle.sla_oracle``."""
from .sla_oracle import *  # noqa: F401,F403
