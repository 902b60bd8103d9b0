"""Float64 CPU oracle for LLA decode (test infrastructure only; see ``oracle.lla``)."""
from .lla import *  # noqa: F401,F403
from .lla import Cfg, Codec  # noqa: F401
