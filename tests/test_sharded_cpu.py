"""The token-sharded long prefill on CPU: the shard plan, ranks emulated one
after another, and two gloo ranks with the all-gather. The per-rank compute is
the oracle, so the sharding logic (halo, scratch state, row assembly, gather)
is checked against the one-shot oracle exactly: every window is computed from
the same numbers either way."""

import os
import socket

import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st
import torch.multiprocessing as mp

from streaming_kv_cache_varlen_b200 import sharded
from workloads import make_inputs


def oracle_call(**kw):
    """One call through the oracle, with the CUDA binding's keyword interface
    (bf16 tensors carried as int16 bits; the states are updated in place)."""
    from oracle.compressor import compressor

    def bits(t):
        return None if t is None else t.numpy().view(np.uint16)

    res = compressor(bits(kw["x"]), kw["kv_state"].numpy(), kw["score_state"].numpy(),
                     kw["kv_block_table"].numpy(), kw["state_block_table"].numpy(),
                     bits(kw["sin"]), bits(kw["cos"]), bits(kw["wkv"]), bits(kw["wgate"]),
                     kw["ape"].numpy(), bits(kw["norm_weight"]), bits(kw["hadamard"]),
                     kw["start_pos"].numpy(), kw["cu_seqlens"].numpy(), kw["ratio"],
                     kw["rope_head_dim"], kw["rotate"])
    kw["kv_state"].copy_(torch.from_numpy(res.kv_state))
    kw["score_state"].copy_(torch.from_numpy(res.score_state))
    return torch.from_numpy(res.out.view(np.int16))


def one_sequence(T, ratio, seed, D=128, H=512, rotate=False, bs=32):
    from oracle import window_row_positions
    inp = make_inputs(name="shard", seed=seed, lengths=[T], start_pos=[0], H=H, D=D,
                      coff=2 if ratio == 4 else 1, ratio=ratio, block_size=bs, rotate=rotate)
    return inp.with_rope(window_row_positions(inp.cu_seqlens, inp.start_pos, ratio))


def t16(a):
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16))


def common_args(inp):
    return dict(x=t16(inp.x), wkv=t16(inp.wkv), wgate=t16(inp.wgate),
                ape=torch.from_numpy(inp.ape), norm_weight=t16(inp.norm_weight),
                hadamard=None if inp.hadamard is None else t16(inp.hadamard),
                sin=t16(inp.sin), cos=t16(inp.cos))


def one_shot(inp):
    from oracle import run_inputs
    return run_inputs(inp)


def tail_rows(inp, res):
    """(positions, kv rows, score rows) of the one-shot call's state tail."""
    T, r = inp.x.shape[0], inp.ratio
    thr = (T // r - (2 if r == 4 else 1) + 1) * r
    pos = np.arange(max(0, thr), T)
    bs = inp.block_size
    rows = inp.kv_block_table[0][pos // bs]
    return pos, res.kv_state[rows, pos % bs], res.score_state[rows, pos % bs]


# ---- the plan -------------------------------------------------------------------

@pytest.mark.parametrize("ratio", [4, 128, 2, 1])
def test_plan_partitions_windows(ratio):
    for T in [0, 1, ratio - 1, ratio, 3 * ratio + 1, 1000, 4096]:
        for world in [1, 2, 3, 8]:
            sh = sharded.plan(T, ratio, world)
            assert len(sh) == world
            nwin = T // ratio
            assert sum(s.n_windows for s in sh) == nwin
            w = 0
            for k, s in enumerate(sh):
                assert s.first_window == w and s.lo == w * ratio
                w += s.n_windows
                assert s.hi == (T if k == world - 1 else w * ratio)
                assert s.x_lo == s.lo - s.skip_rows * ratio
                assert s.skip_rows in (0, 1)
                if ratio != 4 or s.lo == 0 or s.hi == s.lo:
                    assert s.skip_rows == 0
            counts = [s.n_windows for s in sh]
            assert max(counts) - min(counts) <= 1
            if nwin:
                assert sh[-1].n_windows >= 1      # the last rank holds the state tail


# ---- ranks emulated one after another ------------------------------------------

@pytest.mark.parametrize("ratio,T,world,rotate", [(4, 1000, 2, False), (4, 1003, 3, True),
                                                  (4, 8, 4, False), (128, 1100, 3, False),
                                                  (2, 333, 2, False), (4, 7, 3, False)])
def test_emulated_ranks_equal_one_shot(ratio, T, world, rotate):
    emulate_and_check(ratio, T, world, rotate, seed=ratio + T)


@settings(max_examples=25, deadline=None, derandomize=True)
@given(ratio=st.sampled_from([1, 2, 4, 8, 16, 128]), T=st.integers(1, 300), world=st.integers(1, 6),
       rotate=st.booleans(), bs=st.sampled_from([16, 32, 64]), seed=st.integers(0, 1000))
def test_emulated_ranks_equal_one_shot_random(ratio, T, world, rotate, bs, seed):
    """Random lengths, ratios, rank counts and block sizes: the assembled rows
    and the state tail equal the one-shot oracle bit for bit."""
    emulate_and_check(ratio, T, world, rotate, seed=seed, bs=bs)


def emulate_and_check(ratio, T, world, rotate, seed, bs=32):
    inp = one_sequence(T, ratio, seed=seed, rotate=rotate, bs=bs)
    ref = one_shot(inp)
    args = common_args(inp)
    shards = sharded.plan(T, ratio, world)
    rows, locs = [], []
    for s in shards:
        loc = sharded.local_inputs(s, args["x"], args["sin"], args["cos"], ratio, inp.block_size,
                                   inp.wkv.shape[0])
        out = oracle_call(wkv=args["wkv"], wgate=args["wgate"], ape=args["ape"],
                          norm_weight=args["norm_weight"], hadamard=args["hadamard"], ratio=ratio,
                          rope_head_dim=64, rotate=rotate, **loc)
        rows.append(sharded.own_rows(s, out))
        locs.append(loc)
    got = sharded.assemble(shards, rows, T, ratio, rows[-1]).numpy().view(np.uint16)
    assert got.shape == ref.out.shape
    assert np.array_equal(got, ref.out)
    # the state tail comes from the last rank's scratch pool, value for value
    pos, kv_ref, sc_ref = tail_rows(inp, ref)
    last = locs[-1]
    bs = inp.block_size
    lrow = last["kv_block_table"][0].numpy()[pos // bs]
    assert np.array_equal(last["kv_state"].numpy()[lrow, pos % bs], kv_ref)
    assert np.array_equal(last["score_state"].numpy()[lrow, pos % bs], sc_ref)


# ---- two gloo ranks --------------------------------------------------------------

def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, ratio, T, out):
    import datetime

    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        inp = one_sequence(T, ratio, seed=7)
        a = common_args(inp)
        got, loc = sharded.sharded_prefill(a["x"], a["wkv"], a["wgate"], a["ape"], a["norm_weight"],
                                           a["hadamard"], a["sin"], a["cos"], ratio=ratio,
                                           rope_head_dim=64, rotate=False,
                                           block_size=inp.block_size, rank=rank, world=ws,
                                           run_call=oracle_call)
        out[rank] = got.numpy().view(np.uint16).tobytes()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("ratio,T", [(4, 1001), (128, 777)])
def test_two_gloo_ranks_gather_the_one_shot_rows(ratio, T):
    ws = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(ws, _free_port(), ratio, T, out), nprocs=ws, join=True,
                           start_method="spawn")
        res = dict(out)
    ref = one_shot(one_sequence(T, ratio, seed=7)).out
    for r in range(ws):
        got = np.frombuffer(res[r], dtype=np.uint16).reshape(ref.shape)
        assert np.array_equal(got, ref), f"rank {r}"


def oracle_call_bf16(**kw):
    """oracle_call for bf16 tensors (bench.py's inputs) instead of int16 bits."""
    kw = {k: (v.view(torch.int16) if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16 else v)
          for k, v in kw.items()}
    return oracle_call(**kw).view(torch.bfloat16)


def _bench_worker(rank, ws, port, out):
    import datetime
    import types

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=120))
    try:
        args = types.SimpleNamespace(steps=2, warmup=1)
        line, got = bench.bench_sharded(args, ws, rank, torch.device("cpu"), T=600, H=512, D=128,
                                        ratio=4, block_size=32, run_call=oracle_call_bf16)
        out[rank] = (line, got.view(torch.int16).numpy().copy())
    finally:
        dist.destroy_process_group()


def test_bench_sharded_mode_two_gloo_ranks():
    """bench.py --mode sharded's step on two gloo ranks with the oracle as the
    per-rank call: both ranks assemble the one-shot oracle's output exactly, and
    the line carries the contract's keys with strong scaling."""
    ws = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_bench_worker, args=(ws, _free_port(), out), nprocs=ws, join=True,
                           start_method="spawn")
        res = dict(out)
    import bench
    from oracle import run_inputs
    from workloads import Inputs

    inp = bench.sharded_inputs(torch.device("cpu"), 600, 512, 128, 4, seed=1234)
    b = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    one = Inputs(name="shard_bench", ratio=4, coff=2, D=128, rope_head_dim=64, rotate=False, block_size=32,
                 x=b(inp["x"]), wkv=b(inp["wkv"]), wgate=b(inp["wgate"]), ape=inp["ape"].numpy(),
                 norm_weight=b(inp["norm_weight"]), hadamard=None,
                 start_pos=np.zeros(1, np.int32), cu_seqlens=np.array([0, 600], np.int32),
                 kv_state=np.zeros((19, 32, 256), np.float32), score_state=np.zeros((19, 32, 256), np.float32),
                 kv_block_table=np.arange(19, dtype=np.int32)[None], state_block_table=np.arange(19, dtype=np.int32)[None],
                 sin=b(inp["sin"]), cos=b(inp["cos"]))
    ref = run_inputs(one).out
    for rank in range(ws):
        line, got = res[rank]
        assert np.array_equal(got.view(np.uint16), ref), rank
    line = res[0][0]
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "config", "sharded"):
        assert k in line, k
    assert line["scaling"] == "strong" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["sharded"]["windows_per_rank"] == [75, 75]
    assert res[0][0]["ms_per_step"] == res[1][0]["ms_per_step"]   # max over ranks
