"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle."""
from .gen import (  # noqa: F401
    BLOCK_SIZE, CONFIG_NAMES, PREFILL_NAMES, SEED_BASE, ChunkedWorkload, Workload, bits_to_f32,
    build, build_chunked, config, draw_normal_bits, f32_to_bits, poison_byte, prefill_config,
)
