"""CPU oracle (test infrastructure only; see ms_oracle)."""
from .ms_oracle import *  # noqa: F401,F403
from .ms_oracle import OracleModel, OracleCache  # noqa: F401
