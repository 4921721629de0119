"""Oracle package: test infrastructure only (see lowram_oracle's header)."""
from .lowram_oracle import *  # noqa: F401,F403
