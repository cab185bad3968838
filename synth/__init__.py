"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark."""
from .generator import CONFIGS, LayerConfig, gen_layer, gen_slice, gen_tensor, gen_uniform, sweep_configs  # noqa: F401
