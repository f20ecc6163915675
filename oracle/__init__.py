"""fp64 CPU oracle (test infrastructure only; see lora_attn_oracle.py)."""
from .lora_attn_oracle import *  # noqa: F401,F403
from . import lora_attn_oracle as impl  # noqa: F401
