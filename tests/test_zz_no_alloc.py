"""The allocation-free entry point (cmp_compressor_noalloc) gives the same
results as cmp_compressor and as the oracle.

It exists for callers that must not allocate device memory at call time (a
serving engine that reserves all of its memory at start-up, a process running
with the GPU nearly full); its scratch is a fixed array in device memory that
the library image carries. This file is collected last so that a run stopping
at the first failure has run every other test before it. The tests pass alone
in a fresh process and after the other tests (the array may hold an earlier
call's contents).
"""

import ctypes
import dataclasses

import numpy as np
import pytest

from oracle import run_inputs, window_row_positions
from tests.gpu_helpers import (OUT_ATOL, OUT_RTOL, STATE_TOL, assert_out_close, assert_state_close,
                               bits, to_device)
from workloads import bf16_bits_to_f32, make_inputs

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 1 << 20   # the array's size (cmp.h)


def _call(lib, fn_name, a, out):
    import torch
    T, H = a["x"].shape
    B = a["cu_seqlens"].shape[0] - 1
    dims = lib.cmp_dims(B, T, H, a["norm_weight"].shape[0], a["kv_state"].shape[0],
                        a["kv_state"].shape[1], a["kv_block_table"].shape[1])
    p = lambda t: None if t is None else t.data_ptr()
    fn = getattr(lib.lib, fn_name)
    return fn(p(a["x"]), p(a["kv_state"]), p(a["score_state"]), p(a["kv_block_table"]),
              p(a["state_block_table"]), p(a["sin"]), p(a["cos"]), p(a["wkv"]), p(a["wgate"]),
              p(a["ape"]), p(a["norm_weight"]), p(a["hadamard"]), p(a["start_pos"]),
              p(a["cu_seqlens"]), a["ratio"], a["rope_head_dim"], a["rotate"], out.data_ptr(),
              torch.cuda.current_stream().cuda_stream, ctypes.byref(dims))


def _with_rope(inp):
    return inp.with_rope(window_row_positions(inp.cu_seqlens, inp.start_pos, inp.ratio))


def _two_calls_agree(lib, first, second):
    """Runs `first` then `second` (the second continues the state the first left)
    through both entry points; each output and state is checked against the
    other entry point's and against the oracle's."""
    import torch
    reg = to_device(first)
    na = to_device(first)
    okv, osc = first.kv_state, first.score_state
    windows = []
    for step, call in enumerate((first, second)):
        call = dataclasses.replace(_with_rope(call), kv_state=okv, score_state=osc)
        a_reg = to_device(call, kv_state=reg["kv_state"], score_state=reg["score_state"])
        a_na = to_device(call, kv_state=na["kv_state"], score_state=na["score_state"])
        n_out = lib.out_rows(call.B, call.T, call.ratio)
        o_reg = torch.empty((n_out, call.D), dtype=torch.bfloat16, device="cuda")
        o_na = torch.full((n_out, call.D), 7.0, dtype=torch.bfloat16, device="cuda")
        before = (na["kv_state"].cpu().numpy(), na["score_state"].cpu().numpy())
        assert _call(lib, "cmp_compressor", a_reg, o_reg) == 0
        assert _call(lib, "cmp_compressor_noalloc", a_na, o_na) == 0
        assert lib.get_error() == 0
        g = bf16_bits_to_f32(bits(o_na)).astype(np.float64)
        r = bf16_bits_to_f32(bits(o_reg)).astype(np.float64)
        assert np.all(np.abs(g - r) <= OUT_ATOL + OUT_RTOL * np.abs(r)), f"call {step}: outputs differ"
        for k in ("kv_state", "score_state"):
            gs, rs = na[k].cpu().numpy(), reg[k].cpu().numpy()
            assert np.all(np.abs(gs - rs) <= STATE_TOL * np.maximum(np.abs(rs), 1.0)), (step, k)
        # against the oracle, which continues from its own state
        res = run_inputs(call)
        assert_out_close(bits(o_na), res)
        assert_state_close(na["kv_state"].cpu().numpy(), na["score_state"].cpu().numpy(), call, res,
                           *before)
        okv, osc = res.kv_state, res.score_state
        windows.append(len(res.layout.rows))
    return windows


def _split_tokens(both, B, sp):
    """Two calls of one token per request out of a two-token-per-request draw."""
    calls = []
    for step in range(2):
        cu = np.arange(B + 1, dtype=np.int32)
        calls.append(dataclasses.replace(both, x=both.x[step::2], cu_seqlens=cu,
                                         start_pos=(sp + step).astype(np.int32)))
    return calls


def test_c4a_decode_two_calls(lib):
    """32 requests, one token per call, twice: 8 requests complete a window on the
    second call (C4A: D = 512, ratio 4)."""
    B = 32
    rng = np.random.default_rng(21)
    resid = np.concatenate([np.full(8, 2), rng.integers(0, 2, size=B - 8)])
    sp = rng.integers(1, 16384, size=B) * 4 + resid
    both = make_inputs(name="noalloc", seed=21, lengths=[2] * B, start_pos=sp.tolist(), H=4096,
                       D=512, coff=2, ratio=4, block_size=128, rotate=False, lookback=8)
    assert _two_calls_agree(lib, *_split_tokens(both, B, sp)) == [0, 8]


@pytest.mark.parametrize("T", [33, 64])
def test_rotated_c4li_calls(lib, T):
    """The C4Li shape with the Hadamard rotation (D = 128, ratio 4) at 33 and 64
    tokens (the 64-token variants of the projection kernel): a prefill call of
    three sequences, then a continuation call."""
    first_len = [T - 2 * (T // 3), T // 3, T // 3]
    more = [T // 2, T - T // 2 - 3, 3]
    total = [a + b for a, b in zip(first_len, more)]
    whole = make_inputs(name="noalloc_rot", seed=40 + T, lengths=total, start_pos=[0, 5, 2], H=1024,
                        D=128, coff=2, ratio=4, block_size=16, rotate=True, separate_tables=True)
    starts = whole.cu_seqlens[:-1]
    rows1 = np.concatenate([np.arange(s, s + n) for s, n in zip(starts, first_len)])
    rows2 = np.concatenate([np.arange(s + n, s + n + m) for s, n, m in zip(starts, first_len, more)])
    cu1 = np.concatenate([[0], np.cumsum(first_len)]).astype(np.int32)
    cu2 = np.concatenate([[0], np.cumsum(more)]).astype(np.int32)
    first = dataclasses.replace(whole, x=whole.x[rows1], cu_seqlens=cu1)
    second = dataclasses.replace(whole, x=whole.x[rows2], cu_seqlens=cu2,
                                 start_pos=(whole.start_pos + np.asarray(first_len)).astype(np.int32))
    w = _two_calls_agree(lib, first, second)
    assert all(v > 0 for v in w)


def test_ratio128_calls(lib):
    """C128A (coff 1): two sequences, 40 tokens per call, windows completing inside
    the second call."""
    sp = np.array([128 * 3 + 100, 128 * 7 + 90])
    both = make_inputs(name="noalloc_r128", seed=51, lengths=[40, 40], start_pos=sp.tolist(), H=2048,
                       D=512, coff=1, ratio=128, block_size=64, rotate=False, lookback=256)
    first = dataclasses.replace(both, x=both.x[np.r_[0:20, 40:60]],
                                cu_seqlens=np.array([0, 20, 40], np.int32))
    second = dataclasses.replace(both, x=both.x[np.r_[20:40, 60:80]],
                                 cu_seqlens=np.array([0, 20, 40], np.int32),
                                 start_pos=(sp + 20).astype(np.int32))
    assert _two_calls_agree(lib, first, second) == [0, 2]


def _near_limit_b():
    """The largest sequence count whose scratch (error word, three per-sequence
    int32 arrays, fp32 projection rows of 64 tokens x 2 x 1024) fits the array."""
    r = lambda n: (n + 255) // 256 * 256
    proj = r(4 * 64 * 2 * 1024)
    B = 1
    while 256 + r(4 * (B + 2)) + r(4 * (B + 1)) + r(4 * (B + 2)) + proj <= SCRATCH_BYTES:
        B += 1
    return B


def test_scratch_nearly_full(lib):
    """A call whose scratch lands just under the array's size: 64 one-token
    requests spread among tens of thousands of empty sequences, twice in a row."""
    B = _near_limit_b()
    assert B > 40000
    live = np.linspace(0, B - 1, 64).astype(int)
    rng = np.random.default_rng(8)
    sp = np.zeros(B, dtype=np.int64)
    sp[live] = rng.integers(2, 400, size=64) * 4 + np.where(np.arange(64) < 16, 3, rng.integers(0, 3, 64))
    lengths = np.zeros(B, dtype=int)
    lengths[live] = 1
    inp = make_inputs(name="noalloc_full", seed=8, lengths=lengths.tolist(), start_pos=sp.tolist(),
                      H=1024, D=512, coff=2, ratio=4, block_size=128, rotate=False, lookback=8)
    w = _two_calls_agree(lib, inp, inp)  # the same call again: reads only positions before it
    assert w == [16, 16]


def test_bad_table_entry_is_reported(lib):
    """A needed table entry outside the pool: the access is skipped and
    cmp_get_error reports CMP_ERR_DEVICE_INDEX for this entry point too; the next
    call is clean."""
    import torch
    B = 4
    sp = np.array([7, 11, 100, 203])   # residue 3: every request completes a window
    inp = _with_rope(make_inputs(name="noalloc_bad", seed=9, lengths=[1] * B, start_pos=sp.tolist(),
                                 H=1024, D=128, coff=2, ratio=4, block_size=16, rotate=False,
                                 lookback=8))
    assert lib.get_error() == 0
    bad_tbl = inp.kv_block_table.copy()
    bad_tbl[2, sp[2] // 16] = inp.block_num + 5
    a = to_device(dataclasses.replace(inp, kv_block_table=bad_tbl))
    out = torch.empty((lib.out_rows(B, B, 4), 128), dtype=torch.bfloat16, device="cuda")
    assert _call(lib, "cmp_compressor_noalloc", a, out) == 0
    assert lib.get_error() == 5
    assert lib.get_error() == 0       # read and cleared
    a = to_device(inp)
    assert _call(lib, "cmp_compressor_noalloc", a, out) == 0
    assert lib.get_error() == 0
    res = run_inputs(inp)
    assert_out_close(bits(out), res)


def test_rejects_calls_beyond_its_scratch(lib):
    dims = lib.cmp_dims(2, 65, 4096, 512, 4, 128, 4)  # 65 tokens: beyond the 64-token limit
    args = [0x10000] * 14
    st = lib.lib.cmp_compressor_noalloc(*args, 4, 64, False, 0x10000, None, ctypes.byref(dims))
    assert st == 2  # CMP_ERR_INVALID, decided on the host before anything runs
