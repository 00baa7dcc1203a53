"""Seeded synthetic inputs for the MoE-layer workloads (no method arithmetic)."""
from .configs import CONFIGS, BY_NAME, MoEConfig  # noqa: F401
