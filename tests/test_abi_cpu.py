"""The C-ABI library without a GPU: it loads, exports every declared entry point,
rejects bad arguments on the host before launching anything, and its host-side
output-row layout equals the oracle's bit for bit.

Every call below that passes dummy pointers also passes an argument the host
checks reject, so no call here can reach a kernel.
"""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def cmp():
    import streaming_kv_cache_varlen_b200 as m
    return m


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "cmp.h")).read()
    return re.findall(r"CMP_API\s+[\w\s\*]+?\b(cmp_\w+)\s*\(", src)


def test_every_declared_symbol_is_exported(cmp):
    names = declared_symbols()
    assert len(names) >= 12
    lib = ctypes.CDLL(cmp.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_and_kernel_names(cmp):
    assert cmp.lib.cmp_status_string(0) == b"ok"
    for k, name in enumerate(cmp.KERNELS):
        assert cmp.lib.cmp_kernel_name(k).decode() == name
    assert cmp.lib.cmp_kernel_name(99) is None
    assert cmp.set_proj_kernel(0) == 0 and cmp.set_proj_kernel(9) == -1


def test_out_rows(cmp):
    for B, T, r in [(1, 64, 4), (4, 16384, 4), (1, 131072, 128), (32, 32, 4), (0, 0, 4), (3, 5, 2)]:
        assert cmp.out_rows(B, T, r) == min(T, T // r + B)
    assert cmp.out_rows(1, 1, 0) == -1


def test_out_row_layout_matches_oracle(cmp):
    from oracle import layout
    rng = np.random.default_rng(0)
    for _ in range(300):
        ratio = int(rng.choice([2, 4, 8, 16, 32, 64, 128]))
        B = int(rng.integers(1, 9))
        L = rng.integers(0, 3 * ratio + 5, size=B)
        s = rng.integers(0, 5 * ratio, size=B)
        cu = np.concatenate([[0], np.cumsum(L)]).astype(np.int32)
        lay = layout(cu, s, ratio)
        rs, rw = cmp.out_row_layout(cu, s.astype(np.int32), ratio)
        exp_s = np.full(lay.n_out, -1, np.int32)
        exp_w = np.full(lay.n_out, -1, np.int32)
        for row, b, w in lay.rows:
            exp_s[row], exp_w[row] = b, w
        assert np.array_equal(rs, exp_s) and np.array_equal(rw, exp_w)


def test_out_row_layout_rejects_bad_input(cmp):
    with pytest.raises(cmp.CmpError):
        cmp.out_row_layout([0, 5, 3], None, 4)          # not rising
    with pytest.raises(cmp.CmpError):
        cmp.out_row_layout([1, 5], None, 4)             # not from 0
    with pytest.raises(cmp.CmpError):
        cmp.out_row_layout([0, 5], [-1], 4)             # negative start


def _call(cmp, dims, ratio=4, rope=64, rotate=False, had=True, null=None, ptr=0x10000):
    args = [ptr] * 14
    names = ["x", "kv_state", "score_state", "kv_block_table", "state_block_table", "sin", "cos",
             "wkv", "wgate", "ape", "norm_weight", "hadamard", "start_pos", "cu_seqlens"]
    if not had:
        args[11] = None
    if null is not None:
        args[names.index(null)] = None
    d = None if dims is None else ctypes.byref(dims)
    return cmp.lib.cmp_compressor(*args, ratio, rope, rotate, ptr, None, d)


def test_host_checks_reject_before_launch(cmp):
    D = cmp.cmp_dims
    ok = dict(B=2, T=10, H=1024, D=512, block_num=4, block_size=128, table_stride=2)
    assert _call(cmp, None) == 1                                     # dims NULL
    assert _call(cmp, D(**ok), ratio=3) == 3                          # unsupported ratio
    assert _call(cmp, D(**ok), ratio=256) == 3
    assert _call(cmp, D(**ok), rope=32) == 2                          # rope_head_dim != 64
    for k, v in [("D", 256), ("H", 1000), ("H", 0), ("block_size", 0), ("block_size", 2048),
                 ("block_num", 0), ("table_stride", 0), ("B", -1), ("T", -5)]:
        bad = dict(ok)
        bad[k] = v
        assert _call(cmp, D(**bad)) == 2, (k, v)
    bad = dict(ok, B=0)                                               # tokens without sequences
    assert _call(cmp, D(**bad)) == 2
    for name in ["x", "kv_state", "score_state", "kv_block_table", "state_block_table", "sin",
                 "cos", "wkv", "wgate", "ape", "norm_weight", "cu_seqlens"]:
        assert _call(cmp, D(**ok), null=name) == 1, name
    assert _call(cmp, D(**ok), rotate=True, had=False) == 1           # rotate needs hadamard
    assert _call(cmp, D(**ok), ptr=0x10002) == 2                      # misaligned pointers


def _noalloc(cmp, dims, ptrs=None, ptr=0x10000):
    args = [ptr] * 14 if ptrs is None else ptrs
    return cmp.lib.cmp_compressor_noalloc(*args, 4, 64, False, ptr, None, ctypes.byref(dims))


def test_noalloc_host_checks_reject_before_launch(cmp):
    """The allocation-free entry point makes the regular call's host checks,
    the 4-byte alignment of the int32 tables and start_pos included, and rejects
    calls whose scratch would not fit its fixed 1 MiB array."""
    D = cmp.cmp_dims
    ok = dict(B=2, T=10, H=1024, D=512, block_num=4, block_size=128, table_stride=2)
    names = ["x", "kv_state", "score_state", "kv_block_table", "state_block_table", "sin", "cos",
             "wkv", "wgate", "ape", "norm_weight", "hadamard", "start_pos", "cu_seqlens"]
    for name in ("kv_block_table", "state_block_table", "start_pos", "cu_seqlens"):
        ptrs = [0x10000] * 14
        ptrs[names.index(name)] = 0x10001      # misaligned int32 array
        assert _noalloc(cmp, D(**ok), ptrs) == 2, name
    for name in ("x", "wkv", "kv_state"):
        ptrs = [0x10000] * 14
        ptrs[names.index(name)] = 0x10008      # 8 but not 16-byte aligned
        assert _noalloc(cmp, D(**ok), ptrs) == 2, name
    # 64 tokens of 2 x 1024 fp32 projection columns take 512 KiB; the three
    # per-sequence int32 arrays share the rest. 43647 sequences fit, 43648 do not.
    full = dict(ok, T=64, H=4096, D=512)
    assert _noalloc(cmp, D(**dict(full, B=43648))) == 2
    assert _noalloc(cmp, D(**dict(full, T=65))) == 2     # beyond the 64-token limit
    ptrs = [0x10000] * 14
    ptrs[names.index("cu_seqlens")] = 0x10002
    assert _noalloc(cmp, D(**dict(full, B=43647)), ptrs) == 2  # fits; rejected by the alignment


def test_empty_calls_are_noops(cmp):
    D = cmp.cmp_dims
    # nothing to do: OK without touching any pointer (all NULL here)
    args = [None] * 14
    for B, T in [(0, 0), (3, 0)]:
        d = D(B=B, T=T, H=1024, D=128, block_num=1, block_size=16, table_stride=1)
        assert cmp.lib.cmp_compressor(*args, 4, 64, False, None, None, ctypes.byref(d)) == 0


def test_workspace_size(cmp):
    small = cmp.workspace_size(1, 64, 1024, 128, 4, 16, 4, 4)
    big = cmp.workspace_size(1, 131072, 4096, 512, 1024, 128, 1024, 128)
    assert 0 < small < big
    assert big >= 1025 * 512 * 4                # at least the pooled rows of one call
    assert cmp.workspace_size(1, 64, 1000, 128, 4, 16, 4, 4) == 0


def _nsa(cmp, dims, layout=0, dtype=1, cbs=32, stride=16, pbs=128, ptr=0x10000, null=None):
    args = [ptr] * 5 + [ptr]    # input, weight, slot_mapping, act_seq_len, block_table, output_cache
    names = ["input", "weight", "slot_mapping", "act_seq_len", "block_table", "output_cache"]
    if null is not None:
        args[names.index(null)] = None
    d = None if dims is None else ctypes.byref(dims)
    return cmp.lib.cmp_nsa_compress(args[0], args[1], args[2], args[3], args[4], layout, dtype, cbs,
                                    stride, pbs, args[5], None, d)


def test_nsa_host_checks_reject_before_launch(cmp):
    D = cmp.cmp_nsa_dims
    ok = dict(B=4, N=24, D=192, tokens=16, table_stride=4, result_len=512)
    assert _nsa(cmp, None) == 1
    assert _nsa(cmp, D(**ok), dtype=2) == 3
    assert _nsa(cmp, D(**ok), layout=2) == 3
    for kw in [dict(cbs=8), dict(cbs=24), dict(cbs=80), dict(stride=24), dict(cbs=16, stride=32),
               dict(pbs=32), dict(pbs=256)]:
        assert _nsa(cmp, D(**ok), **kw) == 2, kw
    for k, v in [("N", 0), ("N", 65), ("N", 51), ("D", 8), ("D", 24), ("D", 272), ("result_len", 0),
                 ("tokens", 0), ("table_stride", 0), ("B", -1), ("B", 65536),
                 ("tokens", (2**31 - 1) // 128 + 1)]:  # paged rows (tokens x 128) past INT32_MAX
        bad = dict(ok)
        bad[k] = v
        assert _nsa(cmp, D(**bad)) == 2, (k, v)
    for name in ["input", "weight", "slot_mapping", "act_seq_len", "block_table", "output_cache"]:
        assert _nsa(cmp, D(**ok), null=name) == 1, name
    assert _nsa(cmp, D(**ok), ptr=0x10004) == 2          # input / output not 16-byte aligned
    packed_rows = dict(ok, tokens=2**31)                  # packed rows past INT32_MAX
    assert _nsa(cmp, D(**packed_rows), layout=1) == 2
    # packed layout: no block table needed (still rejected here by the misaligned pointer)
    assert _nsa(cmp, D(**ok), layout=1, null="block_table", ptr=0x10004) == 2
    # B == 0: a no-op, no pointer touched
    z = dict(ok, B=0)
    assert cmp.lib.cmp_nsa_compress(None, None, None, None, None, 0, 1, 32, 16, 128, None, None,
                                    ctypes.byref(D(**z))) == 0
