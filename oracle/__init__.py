"""fp64 CPU oracle (test infrastructure only; see ``tsa_oracle``)."""

from .tsa_oracle import attend, attend_rows, clamp_budgets, forward, score, select  # noqa: F401
