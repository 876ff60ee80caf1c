"""FP64 CPU oracle for Sol-Attn / Sol-Attn2 (test infrastructure only; see sol_attn_oracle)."""
from . import sol_attn_oracle  # noqa: F401
