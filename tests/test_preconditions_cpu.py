"""The call's documented preconditions, checked on the host by
``debug_check_tables`` (the library itself never runs it): every table entry a
call needs lies in [0, block_num), and no pool row serves two sequences. Every
workload the tests and the bench use satisfies them; crafted violations are
reported, and padding a call never reads is not."""

import functools

import numpy as np
import pytest

from workloads import make_chunked
from workloads import make_config as _make_config

make_config = functools.lru_cache(maxsize=None)(_make_config)


@pytest.fixture(scope="module")
def cmp():
    import streaming_kv_cache_varlen_b200 as m
    return m


def problems(cmp, i, **over):
    kw = dict(kv_block_table=i.kv_block_table, state_block_table=i.state_block_table,
              cu_seqlens=i.cu_seqlens, start_pos=i.start_pos, ratio=i.ratio, block_size=i.block_size,
              block_num=i.kv_state.shape[0])
    kw.update(over)
    return cmp.debug_check_tables(**kw)


@pytest.mark.parametrize("name", ["c4li_tiny", "c4a_varlen", "c4a_decode"])
def test_workloads_meet_the_preconditions(cmp, name):
    assert problems(cmp, make_config(name)) == []


def test_chunked_calls_meet_the_preconditions(cmp):
    for call in make_chunked().calls:
        assert problems(cmp, call) == []


def test_a_shared_pool_row_is_reported(cmp):
    i = make_config("c4a_varlen")
    # sequences 0 and 1 start at position 0; each writes only its tail block
    e = np.diff(i.cu_seqlens)
    kv = i.kv_block_table.copy()
    kv[1, (e[1] - 1) // i.block_size] = kv[0, (e[0] - 1) // i.block_size]
    out = problems(cmp, i, kv_block_table=kv)
    assert any("kv pool row" in p and "sequences 0 and 1" in p for p in out), out


def test_a_needed_entry_out_of_range_is_reported_and_padding_is_not(cmp):
    i = make_config("c4a_decode")
    # a request that completes a window reads the window's earlier rows from the state
    b = int(np.flatnonzero((i.start_pos + 1) % i.ratio == 0)[0])
    blk = (int(i.start_pos[b]) - 1) // i.block_size
    sc = i.state_block_table.copy()
    sc[b, blk] = -1
    out = problems(cmp, i, state_block_table=sc)
    assert any(f"[{b}][{blk}] = -1" in p for p in out), out
    # padding (entries no call reads) is -1 in this workload and is not reported
    assert (i.kv_block_table == -1).sum() > 0
    assert problems(cmp, i) == []


def test_a_block_past_the_table_is_reported(cmp):
    i = make_config("c4li_tiny")      # 64 tokens from 0, block_size 16: the tail is in block 3
    out = problems(cmp, i, kv_block_table=i.kv_block_table[:, :2])
    assert any("past the table" in p for p in out), out
