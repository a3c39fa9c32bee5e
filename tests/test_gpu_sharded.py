"""The token-sharded long prefill through the CUDA library on one GPU: every
shard of a plan runs as its own call (what each rank of a multi-GPU run does),
the rows are assembled in window order, and the result must match the oracle
of the one-shot call, state tail included. The gather itself is covered by the
gloo test on CPU (tests/test_sharded_cpu.py); only one GPU is available here."""

import numpy as np
import pytest

from oracle import run_inputs, window_row_positions
from streaming_kv_cache_varlen_b200 import sharded
from tests.gpu_helpers import assert_out_close, bf16_dev, bits, dev
from workloads import make_inputs

pytestmark = pytest.mark.gpu


def one_sequence(T, ratio, seed, D, H, rotate, bs=64):
    inp = make_inputs(name="shard", seed=seed, lengths=[T], start_pos=[0], H=H, D=D,
                      coff=2 if ratio == 4 else 1, ratio=ratio, block_size=bs, rotate=rotate)
    return inp.with_rope(window_row_positions(inp.cu_seqlens, inp.start_pos, ratio))


@pytest.mark.parametrize("ratio,T,world,D,rotate", [(4, 4100, 2, 512, False), (4, 3001, 4, 128, True),
                                                    (128, 3077, 3, 512, False), (4, 70, 8, 128, False)])
def test_shards_through_the_library_match_the_one_shot_oracle(lib, ratio, T, world, D, rotate):
    inp = one_sequence(T, ratio, seed=T, D=D, H=1024, rotate=rotate)
    ref = run_inputs(inp)
    b16 = bf16_dev
    x, sin, cos = b16(inp.x), b16(inp.sin), b16(inp.cos)
    common = dict(wkv=b16(inp.wkv), wgate=b16(inp.wgate), ape=dev(inp.ape), norm_weight=b16(inp.norm_weight),
                  hadamard=None if inp.hadamard is None else b16(inp.hadamard), ratio=ratio,
                  rope_head_dim=64, rotate=rotate)
    shards = sharded.plan(T, ratio, world)
    rows, locs = [], []
    for s in shards:
        loc = sharded.local_inputs(s, x, sin, cos, ratio, inp.block_size, inp.wkv.shape[0])
        out = lib.compressor(**common, **loc)
        assert lib.get_error() == 0
        rows.append(sharded.own_rows(s, out))
        locs.append(loc)
    got = bits(sharded.assemble(shards, rows, T, ratio, rows[-1]))
    assert_out_close(got, ref)
    # the state tail, from the last rank's scratch pool
    r, bs = ratio, inp.block_size
    thr = (T // r - (2 if r == 4 else 1) + 1) * r
    pos = np.arange(max(0, thr), T)
    last = locs[-1]
    lrow = last["kv_block_table"][0].cpu().numpy()[pos // bs]
    grow = inp.kv_block_table[0][pos // bs]
    for name in ("kv_state", "score_state"):
        g = last[name].cpu().numpy()[lrow, pos % bs].astype(np.float64)
        e = getattr(ref, name)[grow, pos % bs].astype(np.float64)
        assert (np.abs(g - e) <= 1e-4 * np.maximum(np.abs(e), 1.0)).all(), name
