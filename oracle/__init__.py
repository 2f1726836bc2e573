"""fp64 CPU oracle (test infrastructure only; see ``oracle.ckl_oracle``)."""

from .ckl_oracle import *  # noqa: F401,F403
from .ckl_oracle import __all__  # noqa: F401
