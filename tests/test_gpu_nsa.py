"""NsaCompressWithCache on a B200 against its oracle (oracle/nsa.py): both
layouts, both dtypes, the stride / window sizes of the page's constraints, the
page's example, untouched slots, error reporting."""

import json
import os

import numpy as np
import pytest

from oracle.nsa import nsa_compress, to_f64
from workloads import make_nsa_inputs

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def to_dev(i):
    import torch
    dt = torch.float16 if i.dtype == "fp16" else torch.bfloat16
    b16 = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(dt)
    return dict(input=b16(i.input), weight=b16(i.weight),
                slot_mapping=torch.from_numpy(i.slot_mapping).cuda(),
                act_seq_len=torch.from_numpy(i.act_seq_len).cuda(),
                output_cache=b16(i.output_cache),
                block_table=torch.from_numpy(i.block_table).cuda() if i.layout == "paged" else None)


def gpu_call(cmp, i):
    import torch
    a = to_dev(i)
    cmp.nsa_compress(a["input"], a["weight"], a["slot_mapping"], a["act_seq_len"], a["output_cache"],
                     compress_block_size=i.compress_block_size, compress_stride=i.compress_stride,
                     block_table=a["block_table"], page_block_size=i.page_block_size)
    err = cmp.get_error()
    return a["output_cache"].view(torch.int16).cpu().numpy().view(np.uint16), err


def check(cmp, i):
    ref = nsa_compress(i.input, i.weight, i.slot_mapping, i.act_seq_len, i.block_table, i.output_cache,
                       dtype=i.dtype, compress_block_size=i.compress_block_size,
                       compress_stride=i.compress_stride, page_block_size=i.page_block_size,
                       layout=i.layout)
    got, err = gpu_call(cmp, i)
    assert err == 0
    w = ref.written
    # slots not written: bit for bit the cache before the call
    assert np.array_equal(got[~w], i.output_cache[~w])
    assert_within_fp32_bound(got[w], ref.output_cache[w], ref.abs_sums[w], i.compress_block_size,
                             i.dtype)
    return ref, got


def assert_within_fp32_bound(got_bits, ref_bits, abs_sums, cbs, dtype):
    """Written slots against the exact sum rounded once to the dtype.

    The page fixes fp32 products and an fp32 sum with one round-to-nearest-even
    cast (计算公式 and the kernel description), not the order of the sum. A
    product of two 16-bit values is exact in fp32, and a recursive fp32 sum of
    n terms is within gamma_{n-1} * sum |term| of the exact one (gamma_k =
    k u / (1 - k u), u = 2^-24). Each side's final cast adds at most half a unit
    of the dtype, so |gpu - oracle| <= one unit + gamma_{n-1} * sum |term|."""
    g = to_f64(got_bits, dtype)
    e = to_f64(ref_bits, dtype)
    mant, min_spacing = (10, 2.0 ** -24) if dtype == "fp16" else (7, 2.0 ** -133)
    mag = np.maximum(np.abs(e), np.abs(g))
    ulp = np.maximum(np.exp2(np.floor(np.log2(np.maximum(mag, 1e-300))) - mant), min_spacing)
    u = 2.0 ** -24
    k = cbs - 1
    gamma = k * u / (1 - k * u)
    assert (np.abs(g - e) <= ulp + gamma * abs_sums).all()


@pytest.mark.parametrize("dtype", ["bf16", "fp16"])
@pytest.mark.parametrize("layout", ["paged", "TND"])
@pytest.mark.parametrize("cbs,stride,pbs", [(32, 16, 128), (16, 16, 64), (64, 64, 128), (48, 32, 64),
                                            (64, 16, 64)])
def test_matches_oracle(lib, dtype, layout, cbs, stride, pbs):
    i = make_nsa_inputs(name="nsa", seed=cbs * 7 + stride, B=24, N=24, D=192, compress_block_size=cbs,
                        compress_stride=stride, page_block_size=pbs, dtype=dtype, layout=layout,
                        max_seq_len=512, trigger_fraction=0.6)
    ref, _ = check(lib, i)
    assert ref.written.sum() >= 5


@pytest.mark.parametrize("N,D", [(1, 16), (64, 256), (52, 48), (7, 128)])
def test_head_shapes(lib, N, D):
    i = make_nsa_inputs(name="shape", seed=N + D, B=9, N=N, D=D, compress_block_size=32,
                        compress_stride=32, page_block_size=64, max_seq_len=256, trigger_fraction=0.7)
    check(lib, i)


# Grids whose whole windows do not all fit in the GPU's shared memory at once
# (on 148 SMs), so that the kernel cycles each window's 16-row boxes through a
# ring of fewer buffers: 1536 CTAs with 2 boxes in 1 buffer (the NSA decode
# step of the bench), 1200 CTAs with 4 boxes in 2 buffers, 1320 CTAs with 3
# boxes in 2 buffers (box 2 reuses buffer 0 in its second phase).
@pytest.mark.parametrize("B,N,D,cbs,stride,layout,dtype", [
    (128, 24, 192, 32, 16, "paged", "bf16"),
    (200, 24, 64, 64, 16, "paged", "fp16"),
    (200, 24, 64, 64, 32, "TND", "bf16"),
    (110, 24, 128, 48, 16, "paged", "bf16"),
])
def test_window_ring(lib, B, N, D, cbs, stride, layout, dtype):
    i = make_nsa_inputs(name="ring", seed=B + cbs, B=B, N=N, D=D, compress_block_size=cbs,
                        compress_stride=stride, page_block_size=128, dtype=dtype, layout=layout,
                        max_seq_len=256, trigger_fraction=1.0)
    ref, _ = check(lib, i)
    assert ref.written.sum() == B


def test_pages_example(lib):
    c = json.load(open(os.path.join(GOLDEN, "nsa_example_case.json")))
    import torch
    B, N, D, pbs = c["batch_size"], c["heads_num"], c["heads_dim"], c["page_block_size"]
    per = c["max_seq_len"] // pbs
    h = dict(dtype=torch.float16, device="cuda")
    out = torch.ones((c["result_len"], N, D), **h)
    lib.nsa_compress(torch.ones((per * B, pbs, N, D), **h), torch.ones((c["compress_block_size"], N), **h),
                     torch.tensor(c["slot_mapping"], dtype=torch.int32, device="cuda"),
                     torch.tensor(c["act_seq_len"], dtype=torch.int64, device="cuda"), out,
                     compress_block_size=c["compress_block_size"], compress_stride=c["compress_stride"],
                     block_table=torch.zeros((B, per), dtype=torch.int32, device="cuda"), page_block_size=pbs)
    assert lib.get_error() == 0
    flat = out.reshape(-1).float().cpu().numpy()
    i0 = c["printed_first_index"]
    assert flat[i0:i0 + len(c["expected_printed_values"])].tolist() == c["expected_printed_values"]
    assert (flat[:N * D] == 32.0).all() and (flat[N * D:] == 1.0).all()


def test_repeat_is_bit_identical(lib):
    i = make_nsa_inputs(name="rep", seed=3, B=40, N=8, D=64, compress_block_size=64, compress_stride=16,
                        page_block_size=128, max_seq_len=512, trigger_fraction=1.0)
    a, _ = gpu_call(lib, i)
    b, _ = gpu_call(lib, i)
    assert np.array_equal(a, b)


def test_bad_table_entry_and_slot_are_reported(lib):
    import dataclasses
    i = make_nsa_inputs(name="bad", seed=4, B=3, N=4, D=32, compress_block_size=32, compress_stride=16,
                        page_block_size=64, lengths=[48, 32, 64], max_seq_len=128)
    tbl = i.block_table.copy()
    tbl[0, 0] = i.input.shape[0] + 3           # batch 0 reads page 0 (positions 16..47)
    slots = i.slot_mapping.copy()
    slots[2] = 10_000                          # batch 2's slot is past the cache
    bad = dataclasses.replace(i, block_table=tbl, slot_mapping=slots)
    got, err = gpu_call(lib, bad)
    assert err == 5                            # CMP_ERR_DEVICE_INDEX
    assert lib.get_error() == 0                # cleared by the read
    # batch 1 is still written; batches 0 and 2 are skipped
    ref = nsa_compress(i.input, i.weight, i.slot_mapping, i.act_seq_len, i.block_table, i.output_cache,
                       dtype=i.dtype, compress_block_size=32, compress_stride=16, page_block_size=64)
    s0, s1 = i.slot_mapping[0], i.slot_mapping[1]
    assert np.array_equal(got[s0], i.output_cache[s0])
    assert np.abs(to_f64(got[s1], i.dtype) - to_f64(ref.output_cache[s1], i.dtype)).max() < 0.05


def test_bench_launch_shape(lib):
    """The benchmark's launch: 128 batches, N=24, D=192, bf16, paged (page 128),
    window 32, stride 16, every batch on a compression step (one page per
    batch here to keep the host pool small; the grid and boxes are the same)."""
    i = make_nsa_inputs(name="bench", seed=11, B=128, N=24, D=192, compress_block_size=32, compress_stride=16,
                        page_block_size=128, dtype="bf16", layout="paged", max_seq_len=128,
                        trigger_fraction=1.0)
    ref, _ = check(lib, i)
    assert ref.written.sum() == 128


@pytest.mark.parametrize("layout", ["paged", "TND"])
def test_many_batches(lib, layout):
    """1000 batches: several waves of CTAs on the 148 SMs."""
    i = make_nsa_inputs(name="many", seed=12, B=1000, N=8, D=64, compress_block_size=64, compress_stride=16,
                        page_block_size=64, dtype="fp16", layout=layout, max_seq_len=128, trigger_fraction=0.8)
    ref, _ = check(lib, i)
    assert ref.written.sum() >= 700


def test_packed_rows_of_many_batches(lib):
    """20000 packed batches: every batch's first row comes from the scan kernel
    (chunks of 20 lengths per thread, scanned across the block)."""
    i = make_nsa_inputs(name="scan", seed=13, B=20000, N=1, D=16, compress_block_size=16, compress_stride=16,
                        dtype="bf16", layout="TND", max_seq_len=64, trigger_fraction=0.5)
    ref, _ = check(lib, i)
    assert ref.written.sum() >= 8000


def test_packed_negative_length_is_reported(lib):
    """A negative length makes the rows of every later batch unknown: those
    batches are skipped and reported; earlier ones are still written."""
    import dataclasses
    i = make_nsa_inputs(name="neg", seed=14, B=4, N=2, D=32, compress_block_size=32, compress_stride=16,
                        dtype="fp16", layout="TND", lengths=[48, 40, 32, 64], max_seq_len=64)
    lens = i.act_seq_len.copy()
    lens[1] = -5
    bad = dataclasses.replace(i, act_seq_len=lens)
    got, err = gpu_call(lib, bad)
    assert err == 5                            # CMP_ERR_DEVICE_INDEX
    ref = nsa_compress(i.input, i.weight, i.slot_mapping, i.act_seq_len, i.block_table, i.output_cache,
                       dtype=i.dtype, compress_block_size=32, compress_stride=16, layout="TND")
    s0 = i.slot_mapping[0]
    assert ref.written[s0]
    assert_within_fp32_bound(got[s0], ref.output_cache[s0], ref.abs_sums[s0], 32, i.dtype)
    for b in (2, 3):
        s = i.slot_mapping[b]
        assert np.array_equal(got[s], i.output_cache[s])


@pytest.mark.parametrize("pbs", [64, 128])
def test_long_table_rows(lib, pbs):
    """Table rows wider than 32 pages (the entries are then read one by one
    instead of from the warp's copy of the row), windows deep in the row."""
    i = make_nsa_inputs(name="longrow", seed=15 + pbs, B=6, N=2, D=16, compress_block_size=64,
                        compress_stride=32, page_block_size=pbs, dtype="bf16", layout="paged",
                        max_seq_len=64 * pbs, trigger_fraction=1.0)
    assert i.block_table.shape[1] == 64
    ref, _ = check(lib, i)
    assert ref.written.sum() == 6


def test_largest_heads_and_window(lib):
    """N = 64 heads of D = 256 with a 64-token window: 32 KB per head, one head
    per CTA, the largest shared-memory window a call can ask for."""
    i = make_nsa_inputs(name="maxhead", seed=16, B=4, N=64, D=256, compress_block_size=64, compress_stride=64,
                        page_block_size=128, dtype="fp16", layout="paged", max_seq_len=256, trigger_fraction=1.0)
    ref, _ = check(lib, i)
    assert ref.written.sum() == 4


@pytest.mark.parametrize("layout", ["paged", "TND"])
def test_most_batches(lib, layout):
    """B = 65535, the largest batch count (one grid row per batch)."""
    i = make_nsa_inputs(name="maxb", seed=17, B=65535, N=1, D=16, compress_block_size=16, compress_stride=16,
                        page_block_size=64, dtype="bf16", layout=layout, max_seq_len=64, trigger_fraction=0.5)
    ref, _ = check(lib, i)
    assert ref.written.sum() >= 30000
