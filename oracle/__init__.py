"""CPU oracle of the TACT-KV codec (test infrastructure only; never imported by the product path)."""
from .tactkv_oracle import *  # noqa: F401,F403
from . import tactkv_oracle as core  # noqa: F401
