"""fp64 CPU oracle -- test infrastructure only (see llama_ref.py)."""
from .llama_ref import *  # noqa: F401,F403
