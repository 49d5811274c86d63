"""Float64 CPU oracle (test infrastructure only; see prism_ref's header)."""
from .prism_ref import *  # noqa: F401,F403
from .prism_ref import (OK, ENOCONV, ESTALL, ENONFINITE, POW_INV4, POW_INV2,  # noqa: F401
                        POW_SQRT, PrismOpts, PassInfo)
