"""CPU oracle (test infrastructure only): see moe_ref.py."""
from . import moe_ref  # noqa: F401
