"""Oracle package: test infrastructure only (see wr_oracle's header)."""
from . import wr_oracle  # noqa: F401
