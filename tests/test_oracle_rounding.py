"""The rounding reading of the RMSNorm step: the oracle keeps float64 up to the
one final bf16 rounding, while the PyPTO walk-through's rms_norm helper casts
its fp32 result back to the input dtype (算子级辅助函数). The output tolerance
(|d| <= 2e-2 + 1e-2 |ref|) must hold between the two readings, and the
intermediate rounding must actually change some outputs (else this pins
nothing)."""

import numpy as np
import pytest

from oracle import run_inputs, window_row_positions
from oracle.compressor import bf16_to_f64
from workloads import make_config, make_inputs

OUT_ATOL, OUT_RTOL = 2e-2, 1e-2


def with_rope(inp):
    return inp.with_rope(window_row_positions(inp.cu_seqlens, inp.start_pos, inp.ratio))


CASES = {
    "c4li_tiny": lambda: make_config("c4li_tiny"),
    "c4a_short": lambda: make_inputs(name="c4a_short", seed=21, lengths=[67, 130], start_pos=[0, 5],
                                     H=512, D=512, coff=2, ratio=4, block_size=16, rotate=False),
    "c128a_short": lambda: make_inputs(name="c128a_short", seed=22, lengths=[300], start_pos=[0],
                                       H=512, D=128, coff=1, ratio=128, block_size=64, rotate=True),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_rounding_after_rms_norm_stays_within_the_output_tolerance(name):
    inp = with_rope(CASES[name]())
    a = run_inputs(inp)
    b = run_inputs(inp, round_after_norm=True)
    rows = sorted(r for r, _, _ in a.layout.rows)
    assert rows, "the case must complete windows"
    ea, eb = bf16_to_f64(a.out[rows]), bf16_to_f64(b.out[rows])
    assert np.all(np.abs(ea - eb) <= OUT_ATOL + OUT_RTOL * np.abs(ea))
    assert np.any(a.out[rows] != b.out[rows])
    # everything before the norm is the same computation
    np.testing.assert_array_equal(a.pooled, b.pooled)
    np.testing.assert_array_equal(a.kv_state, b.kv_state)
