"""Parity of the CUDA library with the CPU oracle, on a B200.

Every test runs the library through its C ABI (the ctypes binding) on seeded
inputs from ``workloads`` and compares with ``oracle`` on the same inputs,
under the tolerances in tests/gpu_helpers.py.
"""

import dataclasses
import json
import os

import numpy as np
import pytest

from oracle import run_inputs, window_row_positions
from workloads import make_chunked, make_config, make_inputs, bf16_bits
from tests.gpu_helpers import (assert_out_close, assert_state_close, bits, dev, run, to_device)

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def with_rope(inp):
    return inp.with_rope(window_row_positions(inp.cu_seqlens, inp.start_pos, inp.ratio))


def check(cmp, inp, rows=None):
    out, kv, sc, err = run(cmp, inp)
    assert err == 0, f"device error status {err}"
    res = run_inputs(inp, windows_only=rows)
    assert_out_close(out, res, rows)
    if rows is None:
        assert_state_close(kv, sc, inp, res)
    return out, kv, sc, res


@pytest.fixture(params=[0, 1, 2, 3, 4, 5, 6, 7, 8],
                ids=["auto", "mma", "tcgen05", "decode", "fused", "decode1k", "decodecp", "tcgen05single",
                     "fusedsingle"])
def proj_kernel(request, lib):
    prev = lib.set_proj_kernel(request.param)
    yield request.param
    lib.set_proj_kernel(prev)


# ---- the five workloads ----------------------------------------------------

def test_c4li_tiny_prefill(lib, proj_kernel):
    check(lib, with_rope(make_config("c4li_tiny")))


@pytest.mark.slow
def test_c4a_varlen_prefill(lib):
    check(lib, with_rope(make_config("c4a_varlen")))


def test_c4a_decode(lib, proj_kernel):
    check(lib, with_rope(make_config("c4a_decode")))


@pytest.mark.slow
def test_c128a_128k_prefill(lib):
    inp = with_rope(make_config("c128a_128k"))
    args = to_device(inp)
    kv0 = args["kv_state"].clone()
    sc0 = args["score_state"].clone()
    out = lib.compressor(**args)
    assert lib.get_error() == 0
    o = bits(out)
    assert o.shape == (1025, 512)
    # every one of the 1025 rows against the oracle (a few seconds of CPU work)
    res = run_inputs(inp)
    assert_out_close(o, res)
    assert np.all(o[1024] == 0)
    # e = 131072 is window aligned: no tail, so no state byte may change
    import torch
    assert torch.equal(args["kv_state"], kv0) and torch.equal(args["score_state"], sc0)


@pytest.mark.slow
def test_c4li_chunked_continuation(lib):
    import torch
    ch = make_chunked()
    kv = dev(ch.calls[0].kv_state)
    sc = dev(ch.calls[0].score_state)
    okv, osc = ch.calls[0].kv_state, ch.calls[0].score_state
    per_window = {}
    for c, call in enumerate(ch.calls):
        call = dataclasses.replace(with_rope(call), kv_state=okv, score_state=osc)
        args = to_device(call, kv_state=kv, score_state=sc)
        kv_before, sc_before = kv.cpu().numpy(), sc.cpu().numpy()
        out = bits(lib.compressor(**args))
        assert lib.get_error() == 0
        res = run_inputs(call)   # the oracle continues from its own state
        assert_out_close(out, res)
        assert_state_close(kv.cpu().numpy(), sc.cpu().numpy(), call, res, kv_before, sc_before)
        okv, osc = res.kv_state, res.score_state
        for row, b, w in res.layout.rows:
            per_window[(int(ch.order[c][b]), w)] = out[row]
    one = run_inputs(with_rope(ch.oneshot))
    got = np.zeros_like(one.out)
    for row, b, w in one.layout.rows:
        got[row] = per_window[(b, w)]
    assert len(per_window) == len(one.layout.rows)
    assert_out_close(got, one)
    # the state the chunked calls leave equals the one-shot call's tail
    m = one.written
    d = np.abs(kv.cpu().numpy()[m].astype(np.float64) - one.kv_state[m])
    assert (d <= 1e-4 * np.maximum(np.abs(one.kv_state[m]), 1.0)).all()


# ---- the PyPTO example cases and other ratios -------------------------------

@pytest.mark.parametrize("case", json.load(open(os.path.join(GOLDEN, "pypto_example_cases.json")))["cases"],
                         ids=lambda c: c["name"])
@pytest.mark.parametrize("shift", [0, -2])
def test_pypto_example_cases(lib, case, shift):
    B, S = case["bsz"], case["seq"]
    coff = 2 if case["ratio"] == 4 else 1
    sp = max(0, case["start_pos"] + shift)
    inp = make_inputs(name=case["name"], seed=7, lengths=[S] * B, start_pos=[sp] * B,
                      H=case["H"], D=case["D"], coff=coff, ratio=case["ratio"],
                      block_size=case["block_size"], rotate=case["rotate"], lookback=2 * case["ratio"])
    check(lib, with_rope(inp))


@pytest.mark.parametrize("ratio", [1, 2, 8, 16, 32, 64])
def test_other_ratios(lib, ratio, proj_kernel):
    rng = np.random.default_rng(ratio)
    L = rng.integers(0, 5 * ratio, size=5).tolist()
    sp = rng.integers(0, 3 * ratio, size=5).tolist()
    inp = make_inputs(name="r", seed=ratio, lengths=L, start_pos=sp, H=1024, D=128, coff=1,
                      ratio=ratio, block_size=32, rotate=True)
    check(lib, with_rope(inp))


# ---- edges ----------------------------------------------------------------------

EDGE_CASES = {
    "ragged_tiles": dict(lengths=[1, 129, 300, 0, 77], start_pos=[0, 3, 126, 5, 1], D=512, H=1024,
                         ratio=4, bs=64),
    "c128a_partial_windows": dict(lengths=[200, 1, 130], start_pos=[100, 127, 0], D=512, H=1024,
                                  ratio=128, bs=128),
    "block_size_1": dict(lengths=[9, 6], start_pos=[2, 0], D=128, H=512, ratio=4, bs=1),
    "block_size_1024": dict(lengths=[700, 333], start_pos=[1000, 3], D=128, H=512, ratio=4, bs=1024),
    "far_positions": dict(lengths=[5, 3], start_pos=[(1 << 30) - 3, 2_000_000_001], D=128, H=512,
                          ratio=4, bs=128, lookback=8),
    "d128_ratio128": dict(lengths=[260], start_pos=[0], D=128, H=2048, ratio=128, bs=32),
    "single_token": dict(lengths=[1], start_pos=[3], D=512, H=1024, ratio=4, bs=16),
    "wide_hidden": dict(lengths=[64, 40], start_pos=[0, 0], D=512, H=16384, ratio=4, bs=128),
}


@pytest.fixture(params=[0, 4, 8], ids=["auto", "fused", "fusedsingle"])
def auto_or_fused(request, lib):
    prev = lib.set_proj_kernel(request.param)
    yield request.param
    lib.set_proj_kernel(prev)


@pytest.mark.parametrize("name", sorted(EDGE_CASES))
def test_edge_cases(lib, name, auto_or_fused):
    c = dict(EDGE_CASES[name])
    ratio = c.pop("ratio")
    bs = c.pop("bs")
    inp = make_inputs(name=name, seed=11, coff=2 if ratio == 4 else 1, ratio=ratio, block_size=bs,
                      rotate=c["D"] == 128, **c)
    check(lib, with_rope(inp))


@pytest.mark.parametrize("ratio", [4, 128])
def test_fused_path_history_and_tails(lib, ratio, auto_or_fused):
    """Windows that straddle start_pos (rows from the paged state), tails, zero-length
    sequences and several sequences per tile row, on the fused path."""
    rng = np.random.default_rng(ratio + 5)
    B = 6
    L = [int(v) for v in rng.integers(ratio, 3 * 256, size=B)]
    L[2] = 0
    sp = [int(v) for v in rng.integers(0, 2 * ratio, size=B)]
    inp = make_inputs(name="fh", seed=ratio, lengths=L, start_pos=sp, H=1024,
                      D=512 if ratio == 128 else 128, coff=2 if ratio == 4 else 1, ratio=ratio,
                      block_size=64, rotate=ratio == 4)
    check(lib, with_rope(inp))


# The fused path runs as one kernel (metadata built per CTA, rows finished by the
# last CTA to complete each tile) without rotation and for at most 512 sequences;
# otherwise the scheduler and finish kernels run around it.
FUSED_ONE_KERNEL_CASES = {
    "ratio4_512_sequences": (4, 512, False, 1),
    "ratio4_513_sequences": (4, 513, False, 3),
    "ratio128_512_sequences": (128, 512, False, 1),
    "ratio128_513_sequences": (128, 513, False, 3),
    "ratio4_rotation": (4, 40, True, 3),
}


@pytest.mark.parametrize("name", sorted(FUSED_ONE_KERNEL_CASES))
def test_fused_one_kernel_and_split_forms(lib, name):
    ratio, B, rotate, launches = FUSED_ONE_KERNEL_CASES[name]
    rng = np.random.default_rng(B + ratio)
    hi = 3 * ratio if ratio == 128 else 40
    L = [int(v) for v in rng.integers(0, hi, size=B)]
    sp = [int(v) for v in rng.integers(0, 2 * ratio, size=B)]
    L[0] = 300  # one sequence over two tiles
    inp = make_inputs(name=name, seed=B, lengths=L, start_pos=sp, H=512,
                      D=128, coff=2 if ratio == 4 else 1, ratio=ratio, block_size=32, rotate=rotate)
    prev = lib.set_proj_kernel(4)
    try:
        lib.profile_start()
        check(lib, with_rope(inp))
        launched = lib.profile_stop()
    finally:
        lib.set_proj_kernel(prev)
    assert launched["fused_tcgen05"][1] == 1 and sum(n for _, n in launched.values()) == launches, launched


def test_fused_one_kernel_repeated_calls(lib):
    """The per-tile arrival counters go back to zero: the same call three times,
    then a call with other tiles and channel blocks, agree with the oracle."""
    prev = lib.set_proj_kernel(4)
    try:
        a = with_rope(make_inputs(name="r1", seed=5, lengths=[700, 3, 260], start_pos=[0, 1, 9],
                                  H=512, D=512, coff=2, ratio=4, block_size=64, rotate=False))
        first = check(lib, a)[0]
        for _ in range(2):
            again = check(lib, a)[0]
            assert np.array_equal(first, again)
        b = with_rope(make_inputs(name="r2", seed=6, lengths=[1000, 77], start_pos=[5, 130],
                                  H=512, D=128, coff=1, ratio=128, block_size=128, rotate=False))
        check(lib, b)
        check(lib, a)
    finally:
        lib.set_proj_kernel(prev)


def test_dense_rotation_with_any_matrix(lib):
    inp = make_inputs(name="rot", seed=3, lengths=[40, 21], start_pos=[0, 6], H=1024, D=128,
                      coff=2, ratio=4, block_size=16, rotate=True)
    rng = np.random.default_rng(1)
    inp = dataclasses.replace(inp, hadamard=bf16_bits(rng.standard_normal((128, 128)).astype(np.float32) / 11))
    check(lib, with_rope(inp))


def _rotation(kind, D):
    """hadamard matrices for the rotation tests: the Sylvester matrix with other
    scales (the fast transform applies), and ones that are not scaled Sylvester
    matrices (the dense product applies)."""
    from workloads import sylvester
    h = sylvester(D).astype(np.float32)
    if kind == "sylvester":
        return bf16_bits(h / np.float32(np.sqrt(D)))
    if kind == "scaled_quarter":
        return bf16_bits(h * np.float32(0.25))
    if kind == "negated":
        return bf16_bits(-h / np.float32(np.sqrt(D)))
    if kind == "one_sign_off":       # one entry's sign flipped: not a Sylvester matrix
        h[77, 3] = -h[77, 3]
        return bf16_bits(h / np.float32(np.sqrt(D)))
    if kind == "rows_swapped":       # a Hadamard matrix, but not in Sylvester order
        h[[5, 9]] = h[[9, 5]]
        return bf16_bits(h / np.float32(np.sqrt(D)))
    raise KeyError(kind)


@pytest.mark.parametrize("kind", ["sylvester", "scaled_quarter", "negated", "one_sign_off", "rows_swapped"])
@pytest.mark.parametrize("D", [128, 512])
def test_rotation_by_sylvester_and_other_matrices(lib, proj_kernel, kind, D):
    """The scheduler kernel classifies the hadamard matrix once per call; a scaled
    Sylvester matrix takes the in-register fast Walsh-Hadamard transform (across
    lanes for D = 128, and across warps too for D = 512), any other matrix the
    dense product. Both must match the oracle's dense product."""
    inp = make_inputs(name="rotk", seed=D + len(kind), lengths=[40, 21], start_pos=[0, 6], H=1024, D=D,
                      coff=2, ratio=4, block_size=16, rotate=True)
    inp = dataclasses.replace(inp, hadamard=_rotation(kind, D))
    check(lib, with_rope(inp))


def test_empty_and_noop_calls(lib):
    import torch
    inp = with_rope(make_inputs(name="e", seed=1, lengths=[0, 0], start_pos=[3, 4], H=512, D=128,
                                coff=2, ratio=4, block_size=16, rotate=False, extra_rows=2))
    args = to_device(inp)
    kv0 = args["kv_state"].clone()
    out = lib.compressor(**args)
    assert out.shape == (0, 128) and torch.equal(args["kv_state"], kv0)
    assert lib.get_error() == 0


def test_repeat_is_bit_identical_and_idempotent(lib):
    inp = with_rope(make_inputs(name="d", seed=5, lengths=[333, 91], start_pos=[2, 17], H=2048,
                                D=512, coff=2, ratio=4, block_size=32, rotate=False))
    args = to_device(inp)
    o1 = bits(lib.compressor(**args))
    kv1, sc1 = args["kv_state"].clone(), args["score_state"].clone()
    o2 = bits(lib.compressor(**args))   # state already updated: reads only positions < start
    import torch
    assert np.array_equal(o1, o2)
    assert torch.equal(args["kv_state"], kv1) and torch.equal(args["score_state"], sc1)


def test_projection_kernels_agree(lib):
    """All projection kernels give results within the tolerance of the oracle and,
    for the same kernel, bit-identical repeats."""
    inp = with_rope(make_inputs(name="k", seed=9, lengths=[40, 7, 1, 16], start_pos=[1, 0, 3, 9],
                                H=4096, D=512, coff=2, ratio=4, block_size=128, rotate=False))
    res = run_inputs(inp)
    outs = {}
    for k in (1, 2, 3, 4, 5, 6, 7, 8):
        prev = lib.set_proj_kernel(k)
        try:
            o, kv, sc, err = run(lib, inp)
            o2, _, _, _ = run(lib, inp)
        finally:
            lib.set_proj_kernel(prev)
        assert err == 0
        assert np.array_equal(o, o2)
        assert_out_close(o, res)
        assert_state_close(kv, sc, inp, res)
        outs[k] = o


# The tcgen05 projection runs on CTA pairs (cta_group::2, 256 weight rows per
# pair tile, each CTA holding half of the tile's tokens) unless forced onto
# single CTAs (knob 7). Cases: a ragged last tile whose second half lies past
# T, several tiles per pair (double-buffered accumulators), 2C = 256 / 512 / 1024.
PAIR_CASES = {
    "ragged_tail_d128": ([1500, 1, 1333], [0, 2, 7], 128, 1024, 4),
    "two_tiles_per_pair": ([6000, 5111, 900], [3, 0, 129], 128, 512, 4),
    "d512_ratio4": ([700, 0, 613], [0, 5, 6], 512, 1024, 4),
    "d512_ratio128": ([1100, 400], [100, 0], 512, 1024, 128),
    "d128_ratio1": ([300, 20], [0, 3], 128, 1024, 1),
}


@pytest.mark.parametrize("name", sorted(PAIR_CASES))
@pytest.mark.parametrize("knob", [2, 7], ids=["pairs", "single"])
def test_tcgen05_projection_pairs_and_single(lib, name, knob):
    L, sp, D, H, ratio = PAIR_CASES[name]
    inp = with_rope(make_inputs(name=name, seed=21, lengths=L, start_pos=sp, H=H, D=D,
                                coff=2 if ratio == 4 else 1, ratio=ratio, block_size=64,
                                rotate=D == 128))
    prev = lib.set_proj_kernel(knob)
    try:
        lib.profile_start()
        out = check(lib, inp)[0]
        launched = lib.profile_stop()
        again = run(lib, inp)[0]
    finally:
        lib.set_proj_kernel(prev)
    assert launched["proj_tcgen05"][1] == 1, launched
    assert np.array_equal(out, again)


# ---- the channel-group decode kernel -------------------------------------------------

DECODE_CP_CASES = {
    # name: lengths, start_pos, D, H, ratio, block_size
    "c4a_32way": ([1] * 32, [4 * k + 3 for k in range(32)], 512, 4096, 4, 128),
    "c4a_mixed_starts": ([1] * 24, [k for k in range(24)], 512, 4096, 4, 16),
    "c4a_first_window": ([1, 1, 2, 3], [3, 0, 2, 1], 512, 1024, 4, 8),
    "t64_multi_window": ([30, 17, 9, 8], [2, 0, 5, 61], 512, 2048, 4, 32),
    "t48_ragged": ([20, 0, 27, 1], [6, 3, 0, 9], 128, 1024, 4, 4),
    "ratio1": ([3, 5, 1], [0, 7, 2], 128, 512, 1, 8),
    "ratio2": ([9, 4], [1, 6], 512, 1024, 2, 16),
    "ratio8_tails": ([13, 2, 31], [5, 6, 3], 128, 2048, 8, 16),
    "ratio64": ([1] * 6, [63, 127, 0, 64, 191, 5], 512, 1024, 64, 64),
    "ratio128_overflow": ([1] * 8, [128 * k + 127 for k in range(8)], 512, 1024, 128, 128),
    "single_token": ([1], [3], 512, 1024, 4, 16),
    "wide_hidden": ([16, 5], [3, 0], 512, 16384, 4, 128),
    "many_sequences": ([1] * 64, [4 * k + 3 - (k % 3) for k in range(64)], 128, 512, 4, 8),
}


@pytest.mark.parametrize("name", sorted(DECODE_CP_CASES))
def test_decode_cp_cases(lib, name):
    """Path 6 on windows that straddle start_pos, the first window (no previous
    block), several windows per sequence, tails of every ratio, history rows past
    the prefetch capacity (ratio 128, 8 x 127 state rows), T from 1 to 64."""
    L, sp, D, H, ratio, bs = DECODE_CP_CASES[name]
    inp = with_rope(make_inputs(name=name, seed=13, lengths=L, start_pos=sp, H=H, D=D,
                                coff=2 if ratio == 4 else 1, ratio=ratio, block_size=bs,
                                rotate=False, lookback=2 * ratio))
    prev = lib.set_proj_kernel(6)
    try:
        lib.profile_start()
        check(lib, inp)
        launched = lib.profile_stop()
    finally:
        lib.set_proj_kernel(prev)
    assert launched["decode_cp"][1] == 1, launched


DECODE_CP_ROTATE_CASES = {
    # name: lengths, start_pos, D, H, ratio, block_size, hadamard kind
    "c4li_decode_32way": ([1] * 32, [4 * k + 3 - (k % 4) for k in range(32)], 128, 7168, 4, 128, "sylvester"),
    "c4li_tiny_one_sequence": ([64], [0], 128, 1024, 4, 16, "sylvester"),
    "c4li_any_matrix": ([9, 7, 16], [3, 0, 21], 128, 2048, 4, 16, "one_sign_off"),
    "d512_rotation": ([1] * 24, [4 * k + 3 for k in range(24)], 512, 2048, 4, 64, "scaled_quarter"),
    "ratio8_rotation": ([13, 2, 31], [5, 6, 3], 128, 1024, 8, 16, "negated"),
}


@pytest.mark.parametrize("name", sorted(DECODE_CP_ROTATE_CASES))
def test_decode_cp_with_rotation(lib, name):
    """Path 6 with the Hadamard rotation: each CTA publishes RoPE(y * norm_weight)
    of its channels and forms its output columns from all D of them."""
    L, sp, D, H, ratio, bs, kind = DECODE_CP_ROTATE_CASES[name]
    inp = make_inputs(name=name, seed=17, lengths=L, start_pos=sp, H=H, D=D,
                      coff=2 if ratio == 4 else 1, ratio=ratio, block_size=bs, rotate=True,
                      lookback=2 * ratio)
    inp = with_rope(dataclasses.replace(inp, hadamard=_rotation(kind, D)))
    prev = lib.set_proj_kernel(6)
    try:
        lib.profile_start()
        check(lib, inp)
        launched = lib.profile_stop()
    finally:
        lib.set_proj_kernel(prev)
    assert launched["decode_cp"][1] == 1 and sum(n for _, n in launched.values()) == 1, launched


def test_decode_cp_is_the_automatic_decode_path(lib):
    inp = with_rope(make_config("c4a_decode"))
    lib.profile_start()
    check(lib, inp)
    launched = lib.profile_stop()
    assert launched["decode_cp"][1] == 1 and sum(n for _, n in launched.values()) == 1, launched


# ---- faults are reported, never trapped ------------------------------------------

def test_bad_needed_table_entry_sets_error(lib):
    inp = with_rope(make_inputs(name="bad", seed=2, lengths=[6], start_pos=[9], H=512, D=128,
                                coff=2, ratio=4, block_size=4, rotate=False))
    tbl = inp.kv_block_table.copy()
    tbl[0, 1] = inp.block_num + 5          # block of positions 4..7: the previous window
    out, kv, sc, err = run(lib, dataclasses.replace(inp, kv_block_table=tbl))
    assert err == 5                        # CMP_ERR_DEVICE_INDEX
    assert lib.get_error() == 0            # cleared by the read


def test_unneeded_padding_is_not_read(lib):
    inp = with_rope(make_inputs(name="pad", seed=2, lengths=[6], start_pos=[9], H=512, D=128,
                                coff=2, ratio=4, block_size=4, rotate=False))
    tbl = inp.kv_block_table.copy()
    tbl[0, 0] = -1                         # positions 0..3 are never needed here
    inp = dataclasses.replace(inp, kv_block_table=tbl, state_block_table=tbl.copy())
    check(lib, inp)


def test_bad_cu_seqlens_rejected_on_device(lib, auto_or_fused):
    import torch
    inp = with_rope(make_inputs(name="cu", seed=2, lengths=[6, 10], start_pos=[0, 0], H=512, D=128,
                                coff=2, ratio=4, block_size=16, rotate=False))
    args = to_device(inp)
    args["cu_seqlens"] = torch.tensor([0, 12, 16], dtype=torch.int32, device="cuda")
    args["cu_seqlens"][1] = 20             # not rising to T: the call is rejected
    kv0 = args["kv_state"].clone()
    out = torch.full((lib.out_rows(2, 16, 4), 128), 1.0, dtype=torch.bfloat16, device="cuda")
    lib.compressor(**args, out=out)
    assert lib.get_error() == 5
    assert (bits(out) == 0).all() and torch.equal(args["kv_state"], kv0)


@pytest.mark.parametrize("case", ["c4li_tiny", "c4a_short"])
def test_output_within_tolerance_of_both_rounding_readings(lib, case):
    """The library keeps fp32 to the final bf16 store; the output must be within
    the stated tolerance of the oracle both without and with a bf16 rounding
    after RMSNorm (the PyPTO helper's cast back to the input dtype)."""
    if case == "c4li_tiny":
        inp = make_config("c4li_tiny")
    else:
        inp = make_inputs(name="c4a_short", seed=21, lengths=[67, 130], start_pos=[0, 5], H=512, D=512,
                          coff=2, ratio=4, block_size=16, rotate=False)
    inp = with_rope(inp)
    out, _, _, err = run(lib, inp)
    assert err == 0
    assert_out_close(out, run_inputs(inp))
    assert_out_close(out, run_inputs(inp, round_after_norm=True))


def test_barrier_timeout_is_reported_and_the_next_call_recovers(lib):
    """Failure detection without a GPU fault: a testing knob makes one launch of
    the channel-group decode kernel wait for exchange words of an epoch no CTA
    publishes. Every CTA's bounded wait gives up after about a second, the call
    reports CMP_ERR_TIMEOUT, get_error resets the exchange words, and the next
    call runs normally and matches the oracle."""
    import time
    inp = with_rope(make_config("c4a_decode"))
    prev = lib.set_proj_kernel(6)
    try:
        assert lib.debug_unreachable_barrier(1) == 0
        n0 = lib.launch_count()
        t0 = time.monotonic()
        _, _, _, err = run(lib, inp)
        assert err == 6                                  # CMP_ERR_TIMEOUT
        assert time.monotonic() - t0 < 30
        assert lib.launch_count() - n0 == 1              # the channel-group kernel, once
        assert lib.debug_unreachable_barrier(0) == 0     # the knob was consumed
        check(lib, inp)                                  # the context and the barrier recovered
        check(lib, inp)
    finally:
        lib.debug_unreachable_barrier(0)
        lib.set_proj_kernel(prev)
