"""Seeded synthetic inputs shared by the tests, the oracle checks and the benchmark."""
from .inputs import (  # noqa: F401
    LayerSpec,
    LayerInputs,
    SPECS,
    spec,
    generate,
    bf16_bits_to_f32,
    f32_to_bf16_bits,
)
