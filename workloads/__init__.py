"""Seeded synthetic inputs for the streaming KV-cache Compressor.

This package only draws random numbers and lays them out in the dtypes and
shapes the operator takes. It holds none of the operator's arithmetic, so both
the CPU oracle (``oracle/``) and the CUDA path can be fed from it.
"""

from .synth import (  # noqa: F401
    CONFIG_NAMES,
    Chunked,
    Inputs,
    bf16_bits,
    bf16_bits_to_f32,
    hadamard_bits,
    make_chunked,
    make_config,
    make_inputs,
    rope_tables,
    sylvester,
)
from .nsa import NsaInputs, make_nsa_inputs  # noqa: F401,E402
