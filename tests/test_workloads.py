"""The seeded generators produce the workloads' stated shapes and structure."""

import numpy as np

from workloads import make_chunked, make_config, rope_tables


def test_varlen_prefill_structure():
    w = make_config("c4a_varlen")
    assert w.cu_seqlens.tolist() == [0, 1024, 4025, 9145, 16384]
    assert (w.T, w.H, w.D, w.C, w.ratio, w.coff, w.block_size) == (16384, 4096, 512, 1024, 4, 2, 128)
    assert w.block_num == 8 + 24 + 40 + 57 and w.kv_block_table.shape == (4, 57)
    used = np.sort(w.kv_block_table[w.kv_block_table >= 0])
    assert np.array_equal(used, np.arange(129))          # a permutation of the pool rows
    assert (w.kv_block_table[0, 8:] == -1).all()          # -1 padding past the sequence


def test_decode_structure():
    w = make_config("c4a_decode")
    sp = w.start_pos
    assert w.B == 32 and w.T == 32 and sp.min() >= 4 and sp.max() < 65536
    assert int(((sp + 1) % 4 == 0).sum()) == 8
    assert w.kv_block_table.shape == (32, 512) and w.block_num <= 64
    assert ((w.kv_block_table >= 0).sum(axis=1) <= 2).all()
    again = make_config("c4a_decode")
    assert np.array_equal(again.start_pos, sp) and np.array_equal(again.x, w.x)


def test_tiny_and_chunked():
    w = make_config("c4li_tiny")
    assert (w.T, w.H, w.D, w.rotate, w.block_size) == (64, 1024, 128, True, 16)
    assert w.hadamard.shape == (128, 128)
    ch = make_chunked()
    assert len(ch.calls) == 4 and ch.oneshot.B == 8
    for c, call in enumerate(ch.calls):
        lens = np.diff(call.cu_seqlens)
        assert np.array_equal(lens, ch.chunk_lengths[c][ch.order[c]])
        assert ((1 <= lens) & (lens <= 2048)).all()


def test_rope_tables_half_duplicated():
    c, s = rope_tables([0, 4, 8], 64)
    assert c.shape == (3, 64) and np.array_equal(c[:, :32], c[:, 32:])
    assert (c[0] == 0x3F80).all() and (s[0] == 0).all()
