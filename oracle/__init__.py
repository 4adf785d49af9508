"""fp64 CPU oracle for MLA decode (test infrastructure only; never imported by the library)."""
from .mla_oracle import *  # noqa: F401,F403
