"""Seeded synthetic workloads for MLA decode (shapes, seeds, input tensors only)."""
from .configs import CONFIGS, MLAConfig, shrink  # noqa: F401
from .generate import Workload, make_down_kv_inputs, make_o_proj_inputs, make_workload  # noqa: F401
