"""The allocation-free entry point (cmp_compressor_noalloc) gives the same
results as cmp_compressor.

It exists for callers that must not allocate device memory at call time; its
scratch is a fixed array in device memory that the library image carries.
This file is collected last so that a run stopping at the first failure has
run every other test before it. The test passes alone in a fresh process and
after the other tests (the array may hold an earlier call's contents).
"""

import ctypes

import numpy as np
import pytest

from oracle import window_row_positions
from tests.gpu_helpers import OUT_ATOL, OUT_RTOL, STATE_TOL, bits, to_device
from workloads import bf16_bits_to_f32, make_inputs

pytestmark = pytest.mark.gpu


def _call(lib, fn_name, a, out):
    import torch
    T, H = a["x"].shape
    B = a["cu_seqlens"].shape[0] - 1
    dims = lib.cmp_dims(B, T, H, a["norm_weight"].shape[0], a["kv_state"].shape[0],
                        a["kv_state"].shape[1], a["kv_block_table"].shape[1])
    p = lambda t: None if t is None else t.data_ptr()
    fn = getattr(lib.lib, fn_name)
    st = fn(p(a["x"]), p(a["kv_state"]), p(a["score_state"]), p(a["kv_block_table"]),
            p(a["state_block_table"]), p(a["sin"]), p(a["cos"]), p(a["wkv"]), p(a["wgate"]),
            p(a["ape"]), p(a["norm_weight"]), p(a["hadamard"]), p(a["start_pos"]),
            p(a["cu_seqlens"]), a["ratio"], a["rope_head_dim"], a["rotate"], out.data_ptr(),
            torch.cuda.current_stream().cuda_stream, ctypes.byref(dims))
    assert st == 0, f"{fn_name} returned {st}"


def test_no_alloc_entry_point_matches_regular_one(lib):
    import torch
    B = 32
    rng = np.random.default_rng(21)
    # residue 2: completes a window on the second call; residues 0 / 1: on neither
    resid = np.concatenate([np.full(8, 2), rng.integers(0, 2, size=B - 8)])
    sp = rng.integers(1, 16384, size=B) * 4 + resid
    # two tokens per request, delivered as two calls of one token each
    both = make_inputs(name="noalloc", seed=21, lengths=[2] * B, start_pos=sp.tolist(), H=4096,
                       D=512, coff=2, ratio=4, block_size=128, rotate=False, lookback=8)
    reg = to_device(both)
    na = to_device(both)
    for step in range(2):
        cu = np.arange(B + 1, dtype=np.int32)
        pos = (sp + step).astype(np.int32)
        call = both.__class__(**{**both.__dict__, "x": both.x[step::2], "cu_seqlens": cu,
                                 "start_pos": pos})
        call = call.with_rope(window_row_positions(cu, pos, 4))
        a_reg = to_device(call, kv_state=reg["kv_state"], score_state=reg["score_state"])
        a_na = to_device(call, kv_state=na["kv_state"], score_state=na["score_state"])
        n_out = lib.out_rows(B, B, 4)
        o_reg = torch.empty((n_out, 512), dtype=torch.bfloat16, device="cuda")
        o_na = torch.full((n_out, 512), 7.0, dtype=torch.bfloat16, device="cuda")
        _call(lib, "cmp_compressor", a_reg, o_reg)
        _call(lib, "cmp_compressor_noalloc", a_na, o_na)
        torch.cuda.synchronize()
        g = bf16_bits_to_f32(bits(o_na)).astype(np.float64)
        r = bf16_bits_to_f32(bits(o_reg)).astype(np.float64)
        assert np.all(np.abs(g - r) <= OUT_ATOL + OUT_RTOL * np.abs(r)), f"call {step}: outputs differ"
        for k in ("kv_state", "score_state"):
            gs, rs = na[k].cpu().numpy(), reg[k].cpu().numpy()
            assert np.all(np.abs(gs - rs) <= STATE_TOL * np.maximum(np.abs(rs), 1.0)), (step, k)
        windows = int((np.abs(bits(o_reg)).astype(np.int64).sum(axis=1) != 0).sum())
        assert windows == (8 if step == 1 else 0)


def test_no_alloc_rejects_calls_beyond_its_scratch(lib):
    dims = lib.cmp_dims(2, 65, 4096, 512, 4, 128, 4)  # 65 tokens: beyond the 64-token limit
    args = [0x10000] * 14
    st = lib.lib.cmp_compressor_noalloc(*args, 4, 64, False, 0x10000, None, ctypes.byref(dims))
    assert st == 2  # CMP_ERR_INVALID, decided on the host before anything runs
