"""CPU oracle for the HLWQ Q5 path -- test infrastructure only (see hlwq_oracle)."""

from .hlwq_oracle import *  # noqa: F401,F403
from . import hlwq_oracle  # noqa: F401
