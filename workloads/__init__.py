"""Seeded synthetic workloads for the MoE expert layer (shapes, seeds, value
distributions). Shared by the tests, the benchmark and the oracle checks; holds
none of the layer's arithmetic."""
from .gen import CONFIGS, MoEConfig, make_inputs, bf16_round_np, get_config

__all__ = ["CONFIGS", "MoEConfig", "make_inputs", "bf16_round_np", "get_config"]
