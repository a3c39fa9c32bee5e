"""CPU oracle of the streaming KV-cache Compressor.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package. The CUDA library neither imports nor
links it, and the two share no code; both take their inputs from the seeded
generators in ``workloads``.

* ``oracle.compressor`` — the definition in float64 (numpy), step by step.
* ``oracle.brute`` — a pure-Python restatement from the closed-form formula,
  for tiny inputs, used to pin the former.
* ``oracle.nsa`` — NsaCompressWithCache (the second workload): the weighted sum
  of a batch's last compress_block_size cached tokens, written to its slot,
  with its own brute-force restatement.

Parity status: pinned. No page prints a numeric example of this operator, so
the pins are brute force on tiny inputs, closed forms (equal scores give the
window mean, one dominant score selects its row, masked first window, RMSNorm
unit rms, RoPE identity and pair norms, Hadamard orthogonality) and the
streaming invariants (token by token, chunked and reordered calls equal one
call). See tests/test_oracle_pins.py. One exception, parity unpinned: where
several sequences share a call, the placement of their output rows
(``compressor.layout``) is a reading; no page prints one. The pins fix only what
the pages fix there: the row count min(T, T//ratio + B), zero rows without a
window, one row per request in request order for decode, and window order for
one sequence. ``oracle.nsa`` is pinned by the example
of its page (a closed form on its all-ones inputs), brute force, the trigger
rule and closed forms (tests/test_oracle_nsa.py).
"""

from . import brute, compressor, nsa  # noqa: F401
from .compressor import (  # noqa: F401
    Layout,
    Result,
    bf16_to_f64,
    coff_of,
    f64_to_bf16_bits,
    layout,
    out_rows,
    run_inputs,
    window_row_positions,
)
