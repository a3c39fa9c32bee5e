"""Helpers for the GPU parity tests: move a workload to the device, run the
library through its binding, and compare with the oracle under the stated
tolerances.

Tolerances (written here once and used by every parity test):
  * output rows that hold a window: |gpu - ref| <= 2e-2 + 1e-2 * |ref| per bf16
    element (ref = the oracle's bf16 result);
  * output rows without a window: exactly 0;
  * state slots the call writes: |gpu - ref| <= 1e-4 * max(|ref|, 1);
  * every other state slot: bit-identical to its value before the call.
"""

import numpy as np
import torch

from workloads import bf16_bits_to_f32

OUT_ATOL, OUT_RTOL = 2e-2, 1e-2
STATE_TOL = 1e-4


def bf16_dev(a, device="cuda"):
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(device).view(torch.bfloat16)


def dev(a, device="cuda"):
    if a is None:
        return None
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def to_device(inp, device="cuda", kv_state=None, score_state=None):
    """Keyword arguments of the binding's ``compressor`` for a workloads.Inputs."""
    return dict(x=bf16_dev(inp.x, device),
                kv_state=dev(inp.kv_state, device) if kv_state is None else kv_state,
                score_state=dev(inp.score_state, device) if score_state is None else score_state,
                kv_block_table=dev(inp.kv_block_table, device),
                state_block_table=dev(inp.state_block_table, device),
                sin=bf16_dev(inp.sin, device), cos=bf16_dev(inp.cos, device),
                wkv=bf16_dev(inp.wkv, device), wgate=bf16_dev(inp.wgate, device),
                ape=dev(inp.ape, device), norm_weight=bf16_dev(inp.norm_weight, device),
                hadamard=bf16_dev(inp.hadamard, device), start_pos=dev(inp.start_pos, device),
                cu_seqlens=dev(inp.cu_seqlens, device), ratio=inp.ratio,
                rope_head_dim=inp.rope_head_dim, rotate=inp.rotate)


def bits(t):
    """bf16 tensor -> numpy uint16 bit patterns."""
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def run(cmp, inp, device="cuda"):
    """One call on the device. Returns (out bits, kv_state, score_state, error status)."""
    args = to_device(inp, device)
    out = cmp.compressor(**args)
    err = cmp.get_error()
    return bits(out), args["kv_state"].cpu().numpy(), args["score_state"].cpu().numpy(), err


def assert_out_close(gpu_bits, res, rows=None):
    """Compare output rows (all, or the listed ones) with the oracle's Result."""
    n = res.out.shape[0]
    assert gpu_bits.shape == res.out.shape, (gpu_bits.shape, res.out.shape)
    has = np.zeros(n, dtype=bool)
    for r, _, _ in res.layout.rows:
        has[r] = True
    sel = np.ones(n, dtype=bool) if rows is None else np.isin(np.arange(n), rows)
    empty = sel & ~has
    assert np.all(gpu_bits[empty] == 0), "rows without a window must be exactly 0"
    win = sel & has
    g = bf16_bits_to_f32(gpu_bits[win]).astype(np.float64)
    r = bf16_bits_to_f32(res.out[win]).astype(np.float64)
    assert np.all(np.isfinite(g)), "non-finite output"
    err = np.abs(g - r)
    lim = OUT_ATOL + OUT_RTOL * np.abs(r)
    bad = err > lim
    assert not bad.any(), (f"{int(bad.sum())} of {bad.size} output elements off; "
                           f"max excess {float((err - lim).max()):.3g}")
    return float(err.max()) if err.size else 0.0


def assert_state_close(gpu_kv, gpu_sc, inp, res, before_kv=None, before_sc=None):
    """Written slots within STATE_TOL, untouched slots bit-identical to the device
    state before the call (by default the input's state)."""
    before_kv = inp.kv_state if before_kv is None else before_kv
    before_sc = inp.score_state if before_sc is None else before_sc
    for gpu, before, ref, mask in ((gpu_kv, before_kv, res.kv_state, res.written),
                                   (gpu_sc, before_sc, res.score_state, res.written_score)):
        untouched = ~mask
        assert np.array_equal(gpu[untouched].view(np.uint32), before[untouched].view(np.uint32)), \
            "a state slot the call must not write changed"
        if mask.any():
            d = np.abs(gpu[mask].astype(np.float64) - ref[mask])
            lim = STATE_TOL * np.maximum(np.abs(ref[mask].astype(np.float64)), 1.0)
            assert (d <= lim).all(), f"state off by up to {float((d / lim).max()):.3g} x tolerance"
