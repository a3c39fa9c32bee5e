"""Pins of the CPU oracle against facts the pages and the mathematics fix.

None of these needs a GPU. Each test names the fact it checks; together they
are chosen so that a dropped term, a wrong sign or index, or a transposed
operand anywhere in ``oracle.compressor`` fails at least one of them.
"""

import dataclasses
import json
import math
import os

import numpy as np
import pytest
from hypothesis import assume, given, settings
from hypothesis import strategies as st

import oracle
from oracle import brute
from oracle.compressor import (bf16_to_f64, compressor, f64_to_bf16_bits, layout, out_rows,
                               run_inputs, window_row_positions)
from workloads import bf16_bits, hadamard_bits, make_inputs, sylvester

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(lengths, start_pos, *, ratio=4, D=8, H=16, rope=4, rotate=False, bs=4, seed=0,
         separate=True, x_var=1.0, **kw):
    coff = 2 if ratio == 4 else 1
    inp = make_inputs(name="tiny", seed=seed, lengths=lengths, start_pos=start_pos, H=H, D=D,
                      coff=coff, ratio=ratio, block_size=bs, rotate=rotate, rope_head_dim=rope,
                      separate_tables=separate, x_var=x_var, **kw)
    return inp.with_rope(window_row_positions(inp.cu_seqlens, inp.start_pos, ratio))


def one_hot_x(T, H, cols):
    x = np.zeros((T, H), dtype=np.uint16)
    for t, k in enumerate(cols):
        x[t, k] = 0x3F80
    return x


# ----------------------------------------------------------------------------
# number format
# ----------------------------------------------------------------------------

def test_bf16_rounding_ties_and_specials():
    one = 1.0
    cases = [
        (one, 0x3F80),
        (one + 2.0 ** -8, 0x3F80),            # halfway, even neighbour below
        (one + 3 * 2.0 ** -8, 0x3F82),        # halfway, even neighbour above
        (one + 2.0 ** -8 + 2.0 ** -30, 0x3F81),  # just above halfway
        (-(one + 3 * 2.0 ** -8), 0xBF82),
        (0.0, 0x0000),
        (-0.0, 0x8000),
        (float("inf"), 0x7F80),
        (2.0 ** -130, 0x0008),                # subnormal: 2**-130 = 8 * 2**-133
        (3.0e38 * 2, 0x7F80),                 # overflow
    ]
    for v, bits in cases:
        assert int(f64_to_bf16_bits(np.array([v]))[0]) == bits, v


def test_bf16_rounding_matches_integer_rounding_of_f32():
    # float32 inputs: one RNE rounding by exponent/mantissa arithmetic (oracle) and
    # by integer bit arithmetic (generator) must agree bit for bit.
    rng = np.random.default_rng(5)
    v = (rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))).astype(np.float32)
    assert np.array_equal(f64_to_bf16_bits(v.astype(np.float64)), bf16_bits(v))


# ----------------------------------------------------------------------------
# brute force on tiny inputs
# ----------------------------------------------------------------------------

def _brute(inp):
    lay = layout(inp.cu_seqlens, inp.start_pos, inp.ratio)
    sin = {(b, w): list(inp.sin[r]) for r, b, w in lay.rows}
    cos = {(b, w): list(inp.cos[r]) for r, b, w in lay.rows}
    L = lambda a: None if a is None else a.tolist()
    return lay, brute.compress(L(inp.x), L(inp.kv_state), L(inp.score_state),
                               L(inp.kv_block_table), L(inp.state_block_table), sin, cos,
                               L(inp.wkv), L(inp.wgate), L(inp.ape), L(inp.norm_weight),
                               L(inp.hadamard), L(inp.start_pos), L(inp.cu_seqlens),
                               inp.ratio, inp.rope_head_dim, inp.rotate)


BRUTE_CASES = [
    dict(lengths=[13], start_pos=[0], ratio=4),
    dict(lengths=[5, 0, 9], start_pos=[3, 7, 1], ratio=4),
    dict(lengths=[6, 11], start_pos=[2, 9], ratio=4, rotate=True),
    dict(lengths=[10, 4], start_pos=[0, 5], ratio=2),
    dict(lengths=[12, 3], start_pos=[4, 13], ratio=8),
    dict(lengths=[9], start_pos=[120], ratio=128, bs=16, D=4, H=8),
    dict(lengths=[16], start_pos=[0], ratio=4, D=16, H=8, rope=8, rotate=True, bs=8),
]


@pytest.mark.parametrize("case", BRUTE_CASES)
def test_oracle_matches_brute_force(case):
    _check_against_brute(tiny(**case))


@settings(max_examples=20, deadline=None, derandomize=True)
@given(lengths=st.lists(st.integers(0, 14), min_size=1, max_size=3), data=st.data(),
       ratio=st.sampled_from([1, 2, 4, 8]), rotate=st.booleans(), bs=st.sampled_from([2, 4, 8]),
       seed=st.integers(0, 1000))
def test_oracle_matches_brute_force_random(lengths, data, ratio, rotate, bs, seed):
    """Random tiny varlen calls (empty sequences, mid-window starts, every
    ratio up to 8, with and without rotation): the numpy definition and the
    pure-Python closed form agree."""
    assume(sum(lengths) > 0)
    start_pos = data.draw(st.lists(st.integers(0, 40), min_size=len(lengths), max_size=len(lengths)))
    _check_against_brute(tiny(lengths, start_pos, ratio=ratio, rotate=rotate, bs=bs, seed=seed))


def _check_against_brute(inp):
    res = run_inputs(inp)
    lay, (wins, kv_new, sc_new) = _brute(inp)
    assert len(wins) == len(lay.rows)
    for row, b, w in lay.rows:
        got = res.out_f64[row]
        ref = np.asarray(wins[(b, w)])
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), (row, b, w)
    assert np.array_equal(res.kv_state, np.asarray(kv_new, dtype=np.float32))
    assert np.array_equal(res.score_state, np.asarray(sc_new, dtype=np.float32))
    empty = np.ones(res.layout.n_out, dtype=bool)
    for row, _, _ in lay.rows:
        empty[row] = False
    assert np.all(res.out[empty] == 0)


# ----------------------------------------------------------------------------
# closed forms
# ----------------------------------------------------------------------------

def test_golden_ratio2_closed_form():
    g = json.load(open(os.path.join(GOLDEN, "ratio2_closed_form.json")))
    f = lambda a: bf16_bits(np.asarray(a, dtype=np.float32))
    C = len(g["wkv"])
    res = compressor(np.asarray(g["x_bits"], dtype=np.uint16),
                     np.zeros((1, g["block_size"], C), np.float32),
                     np.zeros((1, g["block_size"], C), np.float32),
                     np.zeros((1, 1), np.int32), np.zeros((1, 1), np.int32),
                     f(g["sin"]), f(g["cos"]), f(g["wkv"]), f(g["wgate"]),
                     np.asarray(g["ape"], np.float32), f(g["norm_weight"]), None,
                     np.asarray(g["start_pos"], np.int32), np.asarray(g["cu_seqlens"], np.int32),
                     g["ratio"], g["rope_head_dim"], g["rotate"])
    assert res.out.tolist() == g["expected_out_bits"]
    assert np.allclose(res.pooled[0], g["expected_pooled_row0"], rtol=0, atol=1e-15)
    assert not res.written.any()


def _equal_score_case(ratio, L, D=8, H=16, seed=1):
    coff = 2 if ratio == 4 else 1
    inp = tiny([L], [0], ratio=ratio, D=D, H=H, seed=seed)
    rng = np.random.default_rng(seed)
    cols = rng.integers(0, H, size=L)
    inp = dataclasses.replace(inp, x=one_hot_x(L, H, cols), wgate=np.zeros_like(inp.wgate),
                              ape=np.zeros_like(inp.ape))
    return inp, cols, coff


@pytest.mark.parametrize("ratio", [4, 8, 128])
def test_equal_scores_give_window_mean(ratio):
    L = 3 * ratio + 1
    inp, cols, coff = _equal_score_case(ratio, L, H=8 if ratio == 128 else 16)
    res = run_inputs(inp)
    W = bf16_to_f64(inp.wkv)      # kv[t][c] = W[c][cols[t]] exactly (one-hot rows)
    D = inp.D
    for row, b, w in res.layout.rows:
        cur = [W[coff * D - D + c if coff == 2 else c][cols[w * ratio:(w + 1) * ratio]]
               for c in range(D)]
        if coff == 2 and w > 0:
            prev = [W[c][cols[(w - 1) * ratio:w * ratio]] for c in range(D)]
            ref = [(prev[c].sum() + cur[c].sum()) / (2 * ratio) for c in range(D)]
        else:
            ref = [cur[c].mean() for c in range(D)]
        assert np.allclose(res.pooled[row], ref, rtol=1e-13, atol=1e-15), (ratio, w)


@pytest.mark.parametrize("ratio", [4, 128])
def test_one_dominant_score_selects_its_row(ratio):
    H = 8
    L = 2 * ratio
    coff = 2 if ratio == 4 else 1
    inp = tiny([L], [0], ratio=ratio, D=8, H=H, bs=16)
    rng = np.random.default_rng(3)
    cols = rng.integers(0, H - 1, size=L)
    star = np.zeros(L, dtype=bool)
    for w in range(L // ratio):          # one token per window carries a +60 score
        star[w * ratio + int(rng.integers(0, ratio))] = True
    x = one_hot_x(L, H, cols)
    x[star, H - 1] = 0x3F80              # second one-hot column H-1 for the starred tokens
    wg = np.zeros_like(inp.wgate)
    wg[:, H - 1] = bf16_bits(np.float32(60.0))
    wk = inp.wkv.copy()
    wk[:, H - 1] = 0
    inp = dataclasses.replace(inp, x=x, wgate=wg, wkv=wk, ape=np.zeros_like(inp.ape))
    res = run_inputs(inp)
    W = bf16_to_f64(inp.wkv)
    D = inp.D
    for row, b, w in res.layout.rows:
        t = w * ratio + int(np.nonzero(star[w * ratio:(w + 1) * ratio])[0][0])
        ref = np.array([W[(D if coff == 2 else 0) + c][cols[t]] for c in range(D)])
        if coff == 2 and w > 0:
            # two dominant rows (previous window's a-half, this window's b-half)
            tp = (w - 1) * ratio + int(np.nonzero(star[(w - 1) * ratio:w * ratio])[0][0])
            ref = (ref + np.array([W[c][cols[tp]] for c in range(D)])) / 2
        assert np.allclose(res.pooled[row], ref, rtol=1e-12, atol=1e-12)


def test_ratio1_pools_each_token_alone():
    # r = 1: every token is its own window, the one-row softmax weight is 1, so the
    # pooled row is the token's kv row ("Triton-Ascend Compressor": with r = 1 only
    # the feature projection and the normalisation remain)
    inp = tiny([5, 3], [7, 0], ratio=1, D=8, H=16)
    res = run_inputs(inp)
    kv, _ = oracle.compressor.project(inp.x, inp.wkv, inp.wgate, inp.ape, [7, 8, 9, 10, 11, 0, 1, 2], 1)
    assert [r for r, _, _ in res.layout.rows] == list(range(8))
    assert np.array_equal(res.pooled, kv.astype(np.float64))
    assert not res.written.any()            # nothing is left for a later call


def test_first_c4a_window_ignores_previous_half():
    inp, cols, _ = _equal_score_case(4, 8)
    res = run_inputs(inp)
    W = bf16_to_f64(inp.wkv)
    D = inp.D
    # window 0: only the 4 b-half rows count (mean of 4, not of 8)
    ref0 = [W[D + c][cols[0:4]].mean() for c in range(D)]
    assert np.allclose(res.pooled[0], ref0, rtol=1e-13)
    # changing the a-half weights leaves window 0 alone and moves window 1
    wk = inp.wkv.copy()
    wk[:D] = bf16_bits(np.float32(3.0))
    res2 = run_inputs(dataclasses.replace(inp, wkv=wk))
    assert np.array_equal(res2.pooled[0], res.pooled[0])
    assert not np.allclose(res2.pooled[1], res.pooled[1])


def test_rmsnorm_unit_rms_with_unit_weight():
    inp = tiny([21], [0], ratio=4, D=8)
    inp = dataclasses.replace(inp, norm_weight=np.full(inp.D, 0x3F80, dtype=np.uint16))
    res = run_inputs(inp)
    for row, _, _ in res.layout.rows:
        y = res.pooled[row]
        ms = np.mean(y * y)
        rms = math.sqrt(np.mean(res.normed[row] ** 2))
        assert abs(rms - math.sqrt(ms / (ms + 1e-6))) < 1e-12


def test_rope_quarter_turn_and_identity():
    inp = tiny([16], [0], ratio=4, D=8, rope=4)
    n = out_rows(1, 16, 4)
    # angle 0: identity on every channel
    c0 = np.full((n, 4), 0x3F80, dtype=np.uint16)
    s0 = np.zeros((n, 4), dtype=np.uint16)
    res = run_inputs(dataclasses.replace(inp, cos=c0, sin=s0))
    assert np.array_equal(res.out_f64, res.normed)
    # angle pi/2 (cos 0, sin 1): each pair (a, b) of the last 4 channels -> (-b, a)
    res = run_inputs(dataclasses.replace(inp, cos=s0, sin=c0))
    z = res.normed
    for row, _, _ in res.layout.rows:
        o = res.out_f64[row]
        assert np.array_equal(o[:4], z[row, :4])
        assert np.array_equal(o[4:], [-z[row, 5], z[row, 4], -z[row, 7], z[row, 6]])


def test_rope_keeps_pair_norms():
    inp = tiny([40], [0], ratio=4, D=8, rope=4)
    ang = np.array([0.3, 1.1, 0.3, 1.1])
    c = np.tile(np.cos(ang), (out_rows(1, 40, 4), 1))
    s = np.tile(np.sin(ang), (out_rows(1, 40, 4), 1))
    # exact float32 values chosen on the unit circle up to bf16 rounding: compare
    # the pair norm change with the closed form cos^2 + sin^2 of the rounded table
    cb, sb = bf16_bits(c.astype(np.float32)), bf16_bits(s.astype(np.float32))
    res = run_inputs(dataclasses.replace(inp, cos=cb, sin=sb))
    k = bf16_to_f64(cb[0]) ** 2 + bf16_to_f64(sb[0]) ** 2
    for row, _, _ in res.layout.rows:
        z, o = res.normed[row], res.out_f64[row]
        for j in range(2):
            nz = z[4 + 2 * j] ** 2 + z[5 + 2 * j] ** 2
            no = o[4 + 2 * j] ** 2 + o[5 + 2 * j] ** 2
            assert abs(no - nz * k[j]) < 1e-12 * max(1.0, nz)


def test_sylvester_orthogonality_and_fwht():
    for d in (2, 8, 128, 512):
        h = sylvester(d).astype(np.int64)
        assert np.array_equal(h @ h.T, d * np.eye(d, dtype=np.int64))
    # fast Walsh-Hadamard butterflies equal the dense product with the Sylvester matrix
    rng = np.random.default_rng(0)
    z = rng.standard_normal(128)
    v = z.copy()
    step = 1
    while step < 128:
        for i in range(0, 128, 2 * step):
            a, b = v[i:i + step].copy(), v[i + step:i + 2 * step].copy()
            v[i:i + step], v[i + step:i + 2 * step] = a + b, a - b
        step *= 2
    assert np.allclose(v, z @ sylvester(128), rtol=0, atol=1e-12)


def test_hadamard_rotation_closed_forms():
    inp = tiny([24], [0], ratio=4, D=8, rope=4, rotate=True)
    base = run_inputs(dataclasses.replace(inp, rotate=False, hadamard=None))
    eye = bf16_bits(np.eye(8, dtype=np.float32))
    res = run_inputs(dataclasses.replace(inp, hadamard=eye))
    assert np.array_equal(res.out_f64, base.out_f64)
    perm = np.random.default_rng(2).permutation(8)
    P = np.zeros((8, 8), dtype=np.float32)
    P[np.arange(8), perm] = 1.0         # z @ P moves channel i to position perm[i]
    res = run_inputs(dataclasses.replace(inp, hadamard=bf16_bits(P)))
    for row, _, _ in res.layout.rows:
        assert np.array_equal(res.out_f64[row][perm], base.out_f64[row])
    res = run_inputs(inp)                # Sylvester / sqrt(8) rounded to bf16
    c = float(bf16_to_f64(hadamard_bits(8))[0, 0])
    for row, _, _ in res.layout.rows:
        ratio = np.linalg.norm(res.out_f64[row]) / np.linalg.norm(base.out_f64[row])
        assert abs(ratio - c * math.sqrt(8)) < 1e-12


# ----------------------------------------------------------------------------
# layout, trigger and the pages' own small examples
# ----------------------------------------------------------------------------

def test_layout_against_trigger_enumeration():
    rng = np.random.default_rng(11)
    for _ in range(200):
        ratio = int(rng.choice([2, 4, 8, 128]))
        B = int(rng.integers(1, 6))
        L = rng.integers(0, 3 * ratio + 3, size=B)
        s = rng.integers(0, 4 * ratio, size=B)
        cu = np.concatenate([[0], np.cumsum(L)])
        lay = layout(cu, s, ratio)
        found = []
        for b in range(B):
            for i in range(int(L[b])):
                if (int(s[b]) + i + 1) % ratio == 0:
                    found.append((b, (int(s[b]) + i) // ratio))
        assert [(b, w) for _, b, w in lay.rows] == found
        rows = [r for r, _, _ in lay.rows]
        assert len(set(rows)) == len(rows)
        assert all(0 <= r < lay.n_out for r in rows)
        assert lay.n_out == min(int(cu[-1]), int(cu[-1]) // ratio + B)


def test_decode_and_single_sequence_rows():
    lay = layout(np.arange(33), np.arange(32) * 5 + 3, 4)
    assert all(r == b for r, b, _ in lay.rows)
    lay = layout([0, 64], [0], 4)
    assert [(r, w) for r, _, w in lay.rows] == [(w, w) for w in range(16)]


def test_ratio2_streaming_example():
    # "r = 2: the first token is only saved; the second one completes the group and
    # produces the compressed output" (Triton-Ascend Compressor article).
    inp = tiny([2], [0], ratio=2, D=8, H=16, bs=4)
    one = run_inputs(inp)
    first = dataclasses.replace(inp, x=inp.x[:1], cu_seqlens=np.array([0, 1], np.int32),
                                sin=inp.sin[:1], cos=inp.cos[:1])
    r1 = run_inputs(first)
    assert r1.layout.rows == [] and np.all(r1.out == 0)
    slot = (inp.kv_block_table[0, 0], 0)
    assert r1.written[slot]
    second = dataclasses.replace(first, x=inp.x[1:], start_pos=np.array([1], np.int32),
                                 kv_state=r1.kv_state, score_state=r1.score_state,
                                 sin=inp.sin[:1], cos=inp.cos[:1])
    r2 = run_inputs(second)
    assert [(b, w) for _, b, w in r2.layout.rows] == [(0, 0)]
    assert np.array_equal(r2.out[0], one.out[0])
    # the pooled value is the two-row softmax written out by hand
    kv, sc = oracle.compressor.project(inp.x, inp.wkv, inp.wgate, inp.ape, [0, 1], 2)
    kv, sc = kv.astype(np.float64), sc.astype(np.float64)
    w0 = 1.0 / (1.0 + np.exp(sc[1] - sc[0]))
    assert np.allclose(r2.pooled[0], w0 * kv[0] + (1 - w0) * kv[1], rtol=1e-13)


def test_update_only_call_writes_state_and_zero_output():
    # "start_pos % ratio + s1 < ratio: no compression; add ape and write each token's
    # kv / score into the state" (PyPTO walk-through, 压缩窗口与状态更新)
    inp = tiny([2, 2], [1, 4], ratio=4, D=8)
    res = run_inputs(inp)
    assert res.layout.rows == [] and np.all(res.out == 0)
    kv, sc = oracle.compressor.project(inp.x, inp.wkv, inp.wgate, inp.ape, [1, 2, 4, 5], 4)
    for t, (b, p) in enumerate([(0, 1), (0, 2), (1, 4), (1, 5)]):
        bs = inp.block_size
        assert np.array_equal(res.kv_state[inp.kv_block_table[b, p // bs], p % bs], kv[t])
        assert np.array_equal(res.score_state[inp.state_block_table[b, p // bs], p % bs], sc[t])
    assert res.written.sum() == 4


def test_state_table_maps_requests_to_pool_rows():
    # "state_block_table = [2, 0, 1]: the three requests use pool rows 2, 0 and 1"
    inp = tiny([3, 3, 3], [0, 0, 0], ratio=4, D=8, bs=8)
    tbl = np.array([[2], [0], [1]], dtype=np.int32)
    inp = dataclasses.replace(inp, kv_block_table=tbl, state_block_table=tbl,
                              kv_state=inp.kv_state[:3], score_state=inp.score_state[:3])
    res = run_inputs(inp)
    kv, _ = oracle.compressor.project(inp.x, inp.wkv, inp.wgate, inp.ape, [0, 1, 2] * 3, 4)
    for req, row in enumerate([2, 0, 1]):
        assert np.array_equal(res.kv_state[row, :3], kv[3 * req:3 * req + 3])


def test_unneeded_padding_is_never_read_and_needed_bad_entry_raises():
    inp = tiny([3], [9], ratio=4, D=8, bs=4)   # positions 9..11: window 2 completes
    tbl = inp.kv_block_table.copy()
    assert tbl[0, 0] >= 0
    tbl[0, 0] = -1                              # block 0 (positions 0..3): never needed
    run_inputs(dataclasses.replace(inp, kv_block_table=tbl, state_block_table=tbl))
    tbl = inp.kv_block_table.copy()
    tbl[0, 1] = -1                              # block 1 holds the previous window (4..7)
    with pytest.raises(IndexError):
        run_inputs(dataclasses.replace(inp, kv_block_table=tbl))


# ----------------------------------------------------------------------------
# streaming invariants
# ----------------------------------------------------------------------------

def _by_window(res, order=None):
    """(request, window) -> (pooled row, output row before the bf16 rounding)."""
    out = {}
    for row, b, w in res.layout.rows:
        req = b if order is None else int(order[b])
        out[(req, w)] = (res.pooled[row], res.out_f64[row])
    return out


def _same(a, b):
    # pooled values are computed from identical float32 rows in the same order, so
    # they agree exactly; the Hadamard product goes through BLAS, whose summation
    # order may depend on how many rows one call holds.
    return np.array_equal(a[0], b[0]) and np.allclose(a[1], b[1], rtol=1e-13, atol=1e-13)


def _split_calls(inp, pieces):
    """Run ``inp`` (all sequences starting at 0) as consecutive calls; pieces[c][b] is
    the number of tokens request b brings to call c. Returns per-window outputs and
    the final states."""
    B = inp.B
    starts = inp.cu_seqlens[:-1]
    done = np.zeros(B, dtype=np.int64)
    kv, sc = inp.kv_state, inp.score_state
    wins = {}
    for c, piece in enumerate(pieces):
        order = np.roll(np.arange(B), c)   # move requests around between calls
        rows = np.concatenate([np.arange(starts[r] + done[r], starts[r] + done[r] + piece[r])
                               for r in order]).astype(np.int64)
        lens = [int(piece[r]) for r in order]
        cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
        sp = np.array([done[r] for r in order], dtype=np.int32)
        call = dataclasses.replace(inp, x=inp.x[rows], cu_seqlens=cu, start_pos=sp,
                                   kv_state=kv, score_state=sc,
                                   kv_block_table=inp.kv_block_table[order],
                                   state_block_table=inp.state_block_table[order])
        call = call.with_rope(window_row_positions(cu, sp, inp.ratio))
        res = run_inputs(call)
        wins.update(_by_window(res, order))
        kv, sc = res.kv_state, res.score_state
        done += np.asarray(piece)
    return wins, kv, sc


@pytest.mark.parametrize("ratio,lengths", [(4, [13, 7, 0]), (8, [19, 9]), (128, [300])])
def test_streaming_equals_one_shot(ratio, lengths):
    D = 8
    inp = tiny(lengths, [0] * len(lengths), ratio=ratio, D=D, H=8 if ratio == 128 else 16,
               bs=16, rotate=ratio == 4)
    one = run_inputs(inp)
    ref = _by_window(one)
    Lmax = max(lengths)
    # token by token
    pieces = [[1 if i < L else 0 for L in lengths] for i in range(Lmax)]
    wins, kv, sc = _split_calls(inp, pieces)
    assert wins.keys() == ref.keys()
    for k in ref:
        assert _same(wins[k], ref[k]), k
    # random chunks
    rng = np.random.default_rng(ratio)
    left = np.asarray(lengths)
    pieces = []
    while left.any():
        p = np.minimum(left, rng.integers(0, 2 * ratio + 3, size=len(lengths)))
        pieces.append(p)
        left = left - p
    wins2, kv2, sc2 = _split_calls(inp, pieces)
    assert wins2.keys() == ref.keys()
    for k in ref:
        assert _same(wins2[k], ref[k]), k
    # the tails the one-shot call keeps are what the split calls keep too
    m, ms = one.written, one.written_score
    assert np.array_equal(kv[m], one.kv_state[m]) and np.array_equal(kv2[m], one.kv_state[m])
    assert np.array_equal(sc[ms], one.score_state[ms]) and np.array_equal(sc2[ms], one.score_state[ms])


@pytest.mark.parametrize("ratio", [4, 128])
def test_tail_rule_is_exactly_what_later_calls_read(ratio):
    coff = 2 if ratio == 4 else 1
    D, H = 8, 8
    for e in range(1, 3 * ratio + 1, 1 if ratio == 4 else 37):
        inp = tiny([e + 2 * ratio], [0], ratio=ratio, D=D, H=H, bs=ratio * 4, seed=e)
        head = dataclasses.replace(inp, x=inp.x[:e], cu_seqlens=np.array([0, e], np.int32))
        head = head.with_rope(window_row_positions(head.cu_seqlens, [0], ratio))
        r1 = run_inputs(head)
        thr = (e // ratio - coff + 1) * ratio
        written = sorted((int(np.nonzero(inp.kv_block_table[0] == r)[0][0]) * inp.block_size + o)
                         for r, o in zip(*np.nonzero(r1.written)))
        assert written == list(range(max(0, thr), e))
        tail = dataclasses.replace(inp, x=inp.x[e:], start_pos=np.array([e], np.int32),
                                   cu_seqlens=np.array([0, 2 * ratio], np.int32),
                                   kv_state=r1.kv_state, score_state=r1.score_state)
        tail = tail.with_rope(window_row_positions(tail.cu_seqlens, [e], ratio))
        ref = run_inputs(tail).out_f64
        # poisoning a slot below the threshold changes nothing later on ...
        for p in range(0, max(0, thr)):
            kv = r1.kv_state.copy()
            kv[inp.kv_block_table[0, p // inp.block_size], p % inp.block_size] = 1e3
            got = run_inputs(dataclasses.replace(tail, kv_state=kv)).out_f64
            assert np.array_equal(got, ref), (e, p)
        # ... and every written slot is read by the next window
        for p in range(max(0, thr), e):
            kv = r1.kv_state.copy()
            kv[inp.kv_block_table[0, p // inp.block_size], p % inp.block_size] = 1e3
            got = run_inputs(dataclasses.replace(tail, kv_state=kv)).out_f64
            assert not np.array_equal(got, ref), (e, p)


def test_reordering_requests_does_not_change_results():
    inp = tiny([9, 6, 14], [3, 0, 5], ratio=4, D=8)
    res = run_inputs(inp)
    order = np.array([2, 0, 1])
    rows = np.concatenate([np.arange(inp.cu_seqlens[r], inp.cu_seqlens[r + 1]) for r in order])
    lens = np.diff(inp.cu_seqlens)[order]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    sp = inp.start_pos[order]
    moved = dataclasses.replace(inp, x=inp.x[rows], cu_seqlens=cu, start_pos=sp,
                                kv_block_table=inp.kv_block_table[order],
                                state_block_table=inp.state_block_table[order])
    moved = moved.with_rope(window_row_positions(cu, sp, 4))
    res2 = run_inputs(moved)
    a, b = _by_window(res), _by_window(res2, order)
    assert a.keys() == b.keys()
    for k in a:
        assert _same(a[k], b[k])
    assert np.array_equal(res.kv_state, res2.kv_state)
    assert np.array_equal(res.score_state, res2.score_state)
