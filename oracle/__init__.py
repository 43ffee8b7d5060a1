"""fp64 CPU oracle (test infrastructure only; see sparse_mla_ref)."""
from .sparse_mla_ref import *  # noqa: F401,F403
from .sparse_mla_ref import lse_rel_err  # noqa: F401
