"""Test infrastructure: the fp64 CPU oracle of the MoE expert layer.

Only tests, the smoke check and the benchmark's CPU-baseline leg use it."""
