"""CPU oracle for the HLWQ Q5 path -- test infrastructure only (see hlwq_oracle)."""

from .hlwq_oracle import *  # noqa: F401,F403
from . import hlwq_oracle  # noqa: F401
from .int4_oracle import *  # noqa: F401,F403,E402
from . import int4_oracle  # noqa: F401,E402
from .kv_oracle import *  # noqa: F401,F403,E402
from . import kv_oracle  # noqa: F401,E402
from .tq3_oracle import *  # noqa: F401,F403,E402
from . import tq3_oracle  # noqa: F401,E402
