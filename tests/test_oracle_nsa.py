"""Pins of the NsaCompressWithCache oracle (CPU): the pages' example, brute force
on tiny inputs, the trigger rule, closed forms (a one-hot weight copies a token,
a power-of-two weight scales exactly) and the paged / packed layouts agreeing."""

import json
import os

import numpy as np
import pytest
from hypothesis import given, settings
from hypothesis import strategies as st

from oracle.nsa import half_to_f64, nsa_compress, nsa_compress_brute, to_f64, triggers
from workloads import make_nsa_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def call(i, **over):
    kw = dict(dtype=i.dtype, compress_block_size=i.compress_block_size,
              compress_stride=i.compress_stride, page_block_size=i.page_block_size, layout=i.layout)
    kw.update(over)
    return nsa_compress(i.input, i.weight, i.slot_mapping, i.act_seq_len, i.block_table,
                        i.output_cache, **kw)


def test_pages_example():
    c = json.load(open(os.path.join(GOLDEN, "nsa_example_case.json")))
    B, N, D = c["batch_size"], c["heads_num"], c["heads_dim"]
    pbs, cbs = c["page_block_size"], c["compress_block_size"]
    per = c["max_seq_len"] // pbs
    one = np.float16(1.0).view(np.uint16)
    inp = np.full((per * B, pbs, N, D), one, dtype=np.uint16)
    w = np.full((cbs, N), one, dtype=np.uint16)
    out0 = np.full((c["result_len"], N, D), one, dtype=np.uint16)
    table = np.zeros((B, per), dtype=np.int32)
    r = nsa_compress(inp, w, c["slot_mapping"], c["act_seq_len"], table, out0, dtype="fp16",
                     compress_block_size=cbs, compress_stride=c["compress_stride"], page_block_size=pbs)
    flat = half_to_f64(r.output_cache).reshape(-1)
    i0 = c["printed_first_index"]
    assert list(flat[i0:i0 + len(c["expected_printed_values"])]) == c["expected_printed_values"]
    assert r.written.tolist() == [True] + [False] * (c["result_len"] - 1)


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("layout", ["paged", "TND"])
@pytest.mark.parametrize("cbs,stride,pbs", [(16, 16, 64), (32, 16, 64), (64, 48, 128), (48, 32, 64)])
def test_brute_force_tiny(dtype, layout, cbs, stride, pbs):
    i = make_nsa_inputs(name="tiny", seed=cbs + stride, B=5, N=3, D=4, compress_block_size=cbs,
                        compress_stride=stride, page_block_size=pbs, dtype=dtype, layout=layout,
                        max_seq_len=200, trigger_fraction=0.7)
    r = call(i)
    ref = nsa_compress_brute(i.input, i.weight, i.slot_mapping, i.act_seq_len, i.block_table,
                             i.output_cache, dtype=dtype, compress_block_size=cbs,
                             compress_stride=stride, page_block_size=pbs, layout=layout)
    assert set(ref) == {(s, n, d) for s in np.nonzero(r.written)[0] for n in range(3) for d in range(4)}
    for (s, n, d), v in ref.items():
        assert r.sums[s, n, d] == v
    assert r.written.sum() >= 1


def test_abs_sums_bound_the_sums():
    """The sums of |product| the GPU tolerance scales with: >= |sum| everywhere,
    equal to the sum when every value is positive, and equal to the brute-force
    sum of |input| * |weight| over the window."""
    import dataclasses
    i = make_nsa_inputs(name="abs", seed=31, B=6, N=3, D=4, compress_block_size=32,
                        compress_stride=16, page_block_size=64, max_seq_len=200, trigger_fraction=1.0)
    r = call(i)
    w = r.written
    assert w.sum() >= 1
    assert (r.abs_sums[w] >= np.abs(r.sums[w])).all()
    # |values|: clear the sign bits, then the sum is its own magnitude
    pos = dataclasses.replace(i, input=i.input & np.uint16(0x7FFF), weight=i.weight & np.uint16(0x7FFF))
    rp = call(pos)
    assert np.array_equal(rp.abs_sums[w], rp.sums[w])
    assert np.array_equal(rp.abs_sums[w], r.abs_sums[w])
    ref = nsa_compress_brute(pos.input, pos.weight, pos.slot_mapping, pos.act_seq_len, pos.block_table,
                             pos.output_cache, dtype="bf16", compress_block_size=32, compress_stride=16,
                             page_block_size=64, layout="paged")
    for (s, n, d), v in ref.items():
        assert r.abs_sums[s, n, d] == v


def test_trigger_rule_and_untouched_slots():
    cbs, stride = 32, 16
    lens = [0, 31, 32, 33, 47, 48, 64, 95, 96, 100]
    i = make_nsa_inputs(name="trig", seed=3, B=len(lens), N=2, D=16, compress_block_size=cbs,
                        compress_stride=stride, page_block_size=64, lengths=lens, max_seq_len=128)
    r = call(i)
    want = [triggers(s, cbs, stride) for s in lens]
    assert want == [False, False, True, False, False, True, True, False, True, False]
    for b, trig in enumerate(want):
        assert r.written[i.slot_mapping[b]] == trig
    untouched = ~r.written
    assert np.array_equal(r.output_cache[untouched], i.output_cache[untouched])


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_one_hot_weight_copies_a_token(dtype):
    cbs = 32
    i = make_nsa_inputs(name="hot", seed=5, B=3, N=4, D=16, compress_block_size=cbs, compress_stride=16,
                        page_block_size=64, dtype=dtype, lengths=[48, 32, 80], max_seq_len=128)
    one = np.float16(1.0).view(np.uint16) if dtype == "fp16" else np.uint16(0x3F80)
    w = np.zeros_like(i.weight)
    hot = [5, 0, 31, 17]           # head n keeps token hot[n] of the window
    for n, j in enumerate(hot):
        w[j, n] = one
    r = nsa_compress(i.input, w, i.slot_mapping, i.act_seq_len, i.block_table, i.output_cache,
                     dtype=dtype, compress_block_size=cbs, compress_stride=16, page_block_size=64)
    for b, s in enumerate(i.act_seq_len):
        for n, j in enumerate(hot):
            p = s - cbs + j
            blk = i.block_table[b][p // 64]
            assert np.array_equal(r.output_cache[i.slot_mapping[b], n], i.input[blk, p % 64, n])


@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_power_of_two_weight_scales_exactly(dtype):
    i = make_nsa_inputs(name="pow2", seed=8, B=6, N=3, D=16, compress_block_size=16, compress_stride=16,
                        page_block_size=64, dtype=dtype, max_seq_len=128, trigger_fraction=1.0)
    r1 = call(i)
    w2 = to_f64(i.weight, dtype) * 2.0
    from oracle.nsa import to_bits
    r2 = nsa_compress(i.input, to_bits(w2, dtype), i.slot_mapping, i.act_seq_len, i.block_table,
                      i.output_cache, dtype=dtype, compress_block_size=16, compress_stride=16,
                      page_block_size=64)
    m = r1.written
    assert m.any()
    assert np.array_equal(to_f64(r2.output_cache[m], dtype), 2.0 * to_f64(r1.output_cache[m], dtype))


def test_paged_and_packed_layouts_agree():
    i = make_nsa_inputs(name="lay", seed=9, B=4, N=2, D=16, compress_block_size=32, compress_stride=32,
                        page_block_size=64, lengths=[32, 64, 96, 70], max_seq_len=128)
    r_paged = call(i)
    # the same tokens packed [T, N, D]
    rows = []
    for b, s in enumerate(i.act_seq_len):
        for p in range(s):
            rows.append(i.input[i.block_table[b][p // 64], p % 64])
    packed = np.stack(rows)
    r_tnd = nsa_compress(packed, i.weight, i.slot_mapping, i.act_seq_len, i.block_table,
                         i.output_cache, dtype=i.dtype, compress_block_size=32, compress_stride=32,
                         layout="TND")
    assert np.array_equal(r_paged.output_cache, r_tnd.output_cache)


@settings(max_examples=20, deadline=None, derandomize=True)
@given(dtype=st.sampled_from(["fp16", "bf16"]), layout=st.sampled_from(["paged", "TND"]),
       cbs=st.sampled_from([16, 32, 48, 64]), stride=st.sampled_from([16, 32, 48, 64]),
       pbs=st.sampled_from([64, 128]), B=st.integers(1, 4), N=st.integers(1, 3),
       seed=st.integers(0, 10_000), frac=st.floats(0.0, 1.0))
def test_brute_force_random(dtype, layout, cbs, stride, pbs, B, N, seed, frac):
    """The definition and its pure-Python restatement agree exactly on random
    small calls, including ones where no batch is on a compression step."""
    if stride > cbs:
        stride = cbs
    i = make_nsa_inputs(name="rand", seed=seed, B=B, N=N, D=4, compress_block_size=cbs,
                        compress_stride=stride, page_block_size=pbs, dtype=dtype, layout=layout,
                        max_seq_len=192, trigger_fraction=frac)
    r = call(i)
    ref = nsa_compress_brute(i.input, i.weight, i.slot_mapping, i.act_seq_len, i.block_table,
                             i.output_cache, dtype=dtype, compress_block_size=cbs,
                             compress_stride=stride, page_block_size=pbs, layout=layout)
    assert set(ref) == {(s, n, d) for s in np.nonzero(r.written)[0] for n in range(N) for d in range(4)}
    for (s, n, d), v in ref.items():
        assert r.sums[s, n, d] == v
    # slots not written keep the cache's bits
    assert np.array_equal(r.output_cache[~r.written], i.output_cache[~r.written])
