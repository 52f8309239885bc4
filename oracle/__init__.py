"""FlashLoop decode-path oracle (test infrastructure only; see flashloop_oracle)."""
from .flashloop_oracle import *  # noqa: F401,F403
from .flashloop_oracle import OracleLayer  # noqa: F401
