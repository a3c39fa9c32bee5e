"""CPU oracle for the streaming KV-cache Compressor (DeepSeek-V4 C4A / C4Li / C128A).

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously correct
definition the CUDA library is checked against. Only ``tests/``, the smoke
check and the CPU-baseline leg of the benchmark may import it; the library
never does, and it shares no code with the library.

Arithmetic: every step runs in float64 on the exact values of the bf16 / fp32
inputs. The two projections are rounded once to float32 (the dtype of the
streaming state, which is also what the pooling reads back), and the output is
rounded once, round-to-nearest-even, to bf16 at the very end.

Sources (page title, then the section or formula used):

* "CANN PyPTO 算子实战: Compressor 长序列 KV Cache 压缩算子" — 主要计算过程,
  参数说明, 返回值说明, 压缩窗口与状态更新, 算子级辅助函数, 数值精度与验证要点.
* "compressor - 算子接口 (torch_extension), CANN 9.2.0-beta.1" — 计算公式 1-5.
* "NPU DeepSeek-V4 Ascend C 融合算子优化" — Compressor 计算公式 (C4A 层, C128A 层).
* "Triton-Ascend Compressor (CANNBot triton-op-generator)" — the streaming /
  state-table semantics (unfinished groups kept across calls, request rows
  found through state_block_table).

Readings taken where the pages are silent or garbled (each one is also in the
design notes): coff = 2 exactly when ratio = 4; the a-half of a coff=2 window
is state columns [0, D) of the previous window and the b-half columns [D, 2D)
of the current one; ape row = position mod ratio; state slot of position p =
(table[b][p // block_size], p % block_size); the state rows written are the
tail rows a later call can still read; output row of the k-th window that
sequence b completes = sum of earlier sequences' capacities min(L, L//ratio+1)
plus k (parity unpinned: no page prints a multi-sequence row placement); interleaved
RoPE pairs (2j, 2j+1) of the last rope_head_dim channels, using table columns j and
rope_head_dim/2 + j.
"""

from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence, Tuple

import numpy as np

RMS_EPS = 1e-6  # rms_norm epsilon ("算子级辅助函数": rms_norm(input, gamma, epsilon=1e-6))


# ----------------------------------------------------------------------------
# number formats
# ----------------------------------------------------------------------------

def bf16_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float64 values."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(v) -> np.ndarray:
    """One round-to-nearest-even rounding of float64 values to bf16 (uint16 bits).

    bf16 keeps 8 significant bits: write v = m * 2**e with 0.5 <= |m| < 1, round
    m * 2**8 to an integer (ties to even), rescale. Below the smallest normal
    (2**-126) the quantum is fixed at 2**-133.
    """
    v = np.asarray(v, dtype=np.float64)
    with np.errstate(over="ignore", invalid="ignore"):
        m, e = np.frexp(v)
        r = np.ldexp(np.rint(m * 256.0) / 256.0, e)
        tiny = np.abs(v) < 2.0 ** -126
        r = np.where(tiny, np.rint(v * 2.0 ** 133) * 2.0 ** -133, r)
        f = r.astype(np.float32)
    bits = (np.ascontiguousarray(f).view(np.uint32) >> 16).astype(np.uint16)
    bits = np.where(np.isnan(v), np.uint16(0x7FC0), bits)
    return bits


def coff_of(ratio: int) -> int:
    """Overlap factor: 2 for ratio 4 (C4A / C4Li), else 1
    ("参数说明": coff = 1 + (ratio == 4))."""
    return 2 if int(ratio) == 4 else 1


def out_rows(B: int, T: int, ratio: int) -> int:
    """Rows of ``out``, ``sin`` and ``cos``: min(T, T // ratio + B) ("返回值说明")."""
    return min(int(T), int(T) // int(ratio) + int(B))


# ----------------------------------------------------------------------------
# output-row layout
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Layout:
    start: np.ndarray   # int64 [B]  first absolute position of each sequence in this call
    length: np.ndarray  # int64 [B]
    cap: np.ndarray     # int64 [B]  rows reserved for the sequence: min(L, L // ratio + 1)
    offset: np.ndarray  # int64 [B+1] first reserved row of each sequence
    first_window: np.ndarray  # int64 [B]  start // ratio
    n_windows: np.ndarray     # int64 [B]  windows completed in this call
    rows: List[Tuple[int, int, int]]  # (out row, sequence, window index) of every window
    n_out: int


def layout(cu_seqlens, start_pos, ratio: int) -> Layout:
    """Which output row holds which (sequence, window).

    A token at absolute position p completes window p // ratio iff
    (p + 1) % ratio == 0 ("数值精度与验证要点": trigger (start_pos + i + 1) % ratio == 0),
    so a sequence covering positions [s, e) completes windows s//ratio .. e//ratio - 1.
    Rows with no completed window stay zero ("返回值说明").
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = cu.shape[0] - 1
    T = int(cu[-1]) if B >= 0 else 0
    s = np.zeros(B, dtype=np.int64) if start_pos is None else np.asarray(start_pos, dtype=np.int64)
    L = cu[1:] - cu[:-1]
    e = s + L
    cap = np.minimum(L, L // ratio + 1)
    off = np.zeros(B + 1, dtype=np.int64)
    off[1:] = np.cumsum(cap)
    w0 = s // ratio
    nw = e // ratio - w0
    rows = []
    for b in range(B):
        for k in range(int(nw[b])):
            rows.append((int(off[b] + k), b, int(w0[b] + k)))
    return Layout(start=s, length=L, cap=cap, offset=off, first_window=w0, n_windows=nw,
                  rows=rows, n_out=out_rows(B, T, ratio))


# ----------------------------------------------------------------------------
# the computation, step by step
# ----------------------------------------------------------------------------

def project(x_rows, wkv, wgate, ape, positions, ratio: int):
    """Dual projection ("计算公式" 1 and 2; "主要计算过程"):
    kv = X Wkv^T, score = X Wgate^T + Ape[position mod ratio].

    Computed in float64 from the exact bf16 values, then rounded once to float32,
    the dtype of kv_state / score_state.
    """
    X = bf16_to_f64(x_rows)
    kv = X @ bf16_to_f64(wkv).T
    sc = X @ bf16_to_f64(wgate).T
    sc = sc + np.asarray(ape, dtype=np.float64)[np.asarray(positions, dtype=np.int64) % ratio]
    return kv.astype(np.float32), sc.astype(np.float32)


def window_positions(windows, ratio: int, coff: int):
    """Absolute positions of the rows pooled for each window.

    coff = 1 (C128A): the ratio rows of the window itself.
    coff = 2 (C4A): ratio rows of the previous window (their a-half, columns
    [0, D)) followed by the ratio rows of the window (their b-half, columns
    [D, 2D)) ("计算公式" 2 and 4: [score^a_(4(i-1)+1 : 4i); score^b_(4i+1 : 4(i+1))]).
    Returns (positions [n, coff*ratio], use_b_half [coff*ratio] bool).
    """
    w = np.asarray(windows, dtype=np.int64).reshape(-1, 1)
    j = np.arange(ratio, dtype=np.int64).reshape(1, -1)
    if coff == 1:
        return w * ratio + j, np.ones(ratio, dtype=bool)
    pos = np.concatenate([(w - 1) * ratio + j, w * ratio + j], axis=1)
    half = np.concatenate([np.zeros(ratio, dtype=bool), np.ones(ratio, dtype=bool)])
    return pos, half


def softmax_pool(K, Z):
    """Per-channel softmax over the window rows, weighting a sum of the kv rows
    ("计算公式" 3-5: S = softmax(score'), C^Comp = [1]_(1 x rows) @ (S ⊙ kv)).

    K, Z: [n, rows, D] float64; Z may hold -inf for masked rows (weight 0).
    The softmax is the stable form (subtract the max, exp, sum, divide) of
    "算子级辅助函数".
    """
    m = Z.max(axis=1, keepdims=True)
    p = np.exp(Z - m)
    return (p * K).sum(axis=1) / p.sum(axis=1)


def rms_norm(y, weight_bits):
    """y / sqrt(mean(y^2) + 1e-6) * weight ("压缩窗口与状态更新", "算子级辅助函数")."""
    g = bf16_to_f64(weight_bits)
    return y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + RMS_EPS) * g


def rope_interleaved(z, cos_bits, sin_bits, rope_head_dim: int):
    """Interleaved RoPE on the last rope_head_dim channels ("压缩窗口与状态更新":
    kv_rope goes through interleaved_rope_2d, rotate_half with transpose/reshape).

    Reading: de-interleave the pairs (2j, 2j+1) into [evens | odds], apply
    u * cos + rotate_half(u) * sin with the row's [rows, rope_head_dim] tables,
    interleave back. Element 2j uses table column j, element 2j+1 column
    rope_head_dim/2 + j.
    """
    D = z.shape[-1]
    h = rope_head_dim // 2
    c = bf16_to_f64(cos_bits)
    s = bf16_to_f64(sin_bits)
    out = z.copy()
    ev = z[:, D - rope_head_dim::2]
    od = z[:, D - rope_head_dim + 1::2]
    out[:, D - rope_head_dim::2] = ev * c[:, :h] - od * s[:, :h]
    out[:, D - rope_head_dim + 1::2] = od * c[:, h:] + ev * s[:, h:]
    return out


def hadamard_rotate(z, hadamard_bits):
    """out @ hadamard, the optional rotation of the C4Li path ("kernel 派发逻辑")."""
    return z @ bf16_to_f64(hadamard_bits)


# ----------------------------------------------------------------------------
# whole calls
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Result:
    out: np.ndarray          # uint16 [n_out, D] bf16 bits
    out_f64: np.ndarray      # float64 [n_out, D] before the bf16 rounding
    pooled: np.ndarray       # float64 [n_out, D] softmax-weighted sums (0 on empty rows)
    normed: np.ndarray       # float64 [n_out, D] after RMSNorm
    kv_state: np.ndarray     # float32, state after the call
    score_state: np.ndarray  # float32
    written: np.ndarray      # bool [block_num, block_size]: kv_state slots this call wrote
    written_score: np.ndarray  # bool [block_num, block_size]: score_state slots written
    layout: Layout


class _SeqRows:
    """Rows (kv, score) of one sequence by absolute position: positions >= start
    come from this call's projections, earlier ones from the paged state
    ("压缩窗口与状态更新": read the window through the page table; the state holds
    what earlier calls projected)."""

    def __init__(self, inp, b, start, length, token0, lazy):
        self.inp, self.b, self.s, self.L, self.t0 = inp, b, int(start), int(length), int(token0)
        self.cache = {}
        if not lazy and self.L > 0:
            pos = self.s + np.arange(self.L, dtype=np.int64)
            self.kv, self.sc = self._project(np.arange(self.L, dtype=np.int64), pos)
        else:
            self.kv = self.sc = None

    def _project(self, idx, pos):
        a = self.inp
        return project(a["x"][self.t0 + idx], a["wkv"], a["wgate"], a["ape"], pos, a["ratio"])

    def current(self, pos):
        """kv / score float32 rows of this call's tokens at absolute positions pos."""
        pos = np.asarray(pos, dtype=np.int64)
        idx = pos - self.s
        if self.kv is not None:
            return self.kv[idx], self.sc[idx]
        need = sorted(set(int(i) for i in idx.ravel()) - set(self.cache))
        if need:
            n = np.asarray(need, dtype=np.int64)
            kv, sc = self._project(n, self.s + n)
            for k, i in enumerate(need):
                self.cache[i] = (kv[k], sc[k])
        C = self.inp["wkv"].shape[0]
        kv = np.empty(idx.shape + (C,), dtype=np.float32)
        sc = np.empty(idx.shape + (C,), dtype=np.float32)
        for j, i in np.ndenumerate(idx):
            kv[j], sc[j] = self.cache[int(i)]
        return kv, sc

    def slot(self, table, pos):
        """Paged slot of absolute positions: (table[b][p // bs], p % bs)."""
        a = self.inp
        bs = a["kv_state"].shape[1]
        blk = np.asarray(pos, dtype=np.int64) // bs
        if blk.size and (blk.max() >= table.shape[1] or blk.min() < 0):
            raise IndexError(f"sequence {self.b}: block index beyond the block table")
        rows = table[self.b][blk].astype(np.int64)
        nb = a["kv_state"].shape[0]
        if rows.size and (rows.min() < 0 or rows.max() >= nb):
            raise IndexError(f"sequence {self.b}: block table entry outside [0, block_num)")
        return rows, np.asarray(pos, dtype=np.int64) % bs

    def rows(self, pos):
        """(K, Z) float64 [..., C] for absolute positions pos (all >= 0)."""
        a = self.inp
        pos = np.asarray(pos, dtype=np.int64)
        C = a["wkv"].shape[0]
        K = np.empty(pos.shape + (C,), dtype=np.float64)
        Z = np.empty(pos.shape + (C,), dtype=np.float64)
        cur = pos >= self.s
        if cur.any():
            kv, sc = self.current(pos[cur])
            K[cur], Z[cur] = kv, sc
        hist = ~cur
        if hist.any():
            r, o = self.slot(a["kv_block_table"], pos[hist])
            K[hist] = a["kv_state"][r, o]
            r, o = self.slot(a["state_block_table"], pos[hist])
            Z[hist] = a["score_state"][r, o]
        return K, Z


def _as_dict(**kw):
    return kw


def _pool_windows(seq: _SeqRows, windows, ratio, coff, D):
    """Softmax-pooled y [n, D] of the given windows of one sequence."""
    pos, use_b = window_positions(windows, ratio, coff)
    C = coff * D
    # First window of a sequence: the previous window does not exist; its rows
    # count as kv = 0, score = -inf ("压缩窗口与状态更新": 用 0 和 -inf 填充前序窗口).
    valid = pos >= 0
    K = np.zeros(pos.shape + (C,), dtype=np.float64)
    Z = np.full(pos.shape + (C,), -np.inf, dtype=np.float64)
    if valid.any():
        K[valid], Z[valid] = seq.rows(pos[valid])
    if coff == 2:
        K = np.where(use_b[None, :, None], K[..., D:], K[..., :D])
        Z = np.where(use_b[None, :, None], Z[..., D:], Z[..., :D])
    return softmax_pool(K, Z)


def _check_args(a):
    ratio = int(a["ratio"])
    coff = coff_of(ratio)
    T, H = a["x"].shape
    C = a["wkv"].shape[0]
    if C % coff:
        raise ValueError("wkv rows must be coff * D")
    D = C // coff
    if a["wgate"].shape != (C, H) or a["wkv"].shape != (C, H):
        raise ValueError("wkv / wgate must be [coff*D, H]")
    if a["ape"].shape != (ratio, C):
        raise ValueError("ape must be [ratio, coff*D]")
    if a["kv_state"].shape[2] != C or a["score_state"].shape != a["kv_state"].shape:
        raise ValueError("states must be [block_num, block_size, coff*D]")
    if a["rotate"] and a["hadamard"] is None:
        raise ValueError("rotate needs a hadamard matrix")
    return ratio, coff, T, H, C, D


def compressor(x, kv_state, score_state, kv_block_table, state_block_table, sin, cos,
               wkv, wgate, ape, norm_weight, hadamard, start_pos, cu_seqlens,
               ratio, rope_head_dim, rotate, *, windows_only: Optional[Sequence[int]] = None,
               write_state: bool = True, chunk: int = 512, round_after_norm: bool = False) -> Result:
    """One call of the Compressor, with the argument order of the pages' prototype
    ("函数原型": x, kv_state, score_state, kv_block_table, state_block_table, sin, cos,
    wkv, wgate, ape, weight, hadamard, start_pos, ratio, rope_head_dim, rotate),
    plus cu_seqlens for packed variable-length input.

    x is [T, H] packed: sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1 at
    absolute positions start_pos[b] + i. ``windows_only`` restricts the work to the
    listed output rows (for spot checks of very large calls); other rows then
    come back as NaN in the float arrays and 0 in ``out``. ``write_state=False``
    skips the state update.

    ``round_after_norm`` rounds the RMSNorm result to bf16 before RoPE and the
    rotation: the PyPTO walk-through's rms_norm helper works in fp32 and casts its
    result back to the input dtype (算子级辅助函数). The default keeps float64 up to
    the one final rounding. The output tolerance is meant to hold for either
    reading.
    """
    a = _as_dict(x=np.asarray(x), kv_state=np.asarray(kv_state, dtype=np.float32),
                 score_state=np.asarray(score_state, dtype=np.float32),
                 kv_block_table=np.asarray(kv_block_table, dtype=np.int64),
                 state_block_table=np.asarray(state_block_table, dtype=np.int64),
                 wkv=np.asarray(wkv), wgate=np.asarray(wgate),
                 ape=np.asarray(ape, dtype=np.float32), ratio=int(ratio), rotate=bool(rotate),
                 hadamard=None if hadamard is None else np.asarray(hadamard))
    ratio, coff, T, H, C, D = _check_args(a)
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    if cu[0] != 0 or np.any(np.diff(cu) < 0) or cu[-1] != T:
        raise ValueError("cu_seqlens must rise from 0 to T")
    B = cu.shape[0] - 1
    sp = np.zeros(B, dtype=np.int64) if start_pos is None else np.asarray(start_pos, dtype=np.int64)
    if np.any(sp < 0):
        raise ValueError("start_pos must be >= 0")
    lay = layout(cu, sp, ratio)
    n_out = lay.n_out
    fill = np.nan if windows_only is not None else 0.0
    pooled = np.full((n_out, D), fill)
    want = None if windows_only is None else set(int(r) for r in windows_only)

    seqs = [_SeqRows(a, b, sp[b], lay.length[b], cu[b], lazy=want is not None) for b in range(B)]
    rows_by_seq = {}
    for (row, b, w) in lay.rows:
        if want is None or row in want:
            rows_by_seq.setdefault(b, []).append((row, w))
    if want is not None:
        for r in want:
            if r not in {row for row, _, _ in lay.rows} and 0 <= r < n_out:
                pooled[r] = 0.0
    for b, lst in rows_by_seq.items():
        for i in range(0, len(lst), chunk):
            part = lst[i:i + chunk]
            y = _pool_windows(seqs[b], [w for _, w in part], ratio, coff, D)
            pooled[[r for r, _ in part]] = y

    has = np.zeros(n_out, dtype=bool)
    for (row, b, w) in lay.rows:
        has[row] = True
    sel = has & ~np.isnan(pooled[:, 0])
    normed = np.where(has[:, None], pooled, 0.0) if want is None else pooled.copy()
    out_f = normed.copy()
    if sel.any():
        z = rms_norm(pooled[sel], norm_weight)
        if round_after_norm:
            z = bf16_to_f64(f64_to_bf16_bits(z))
        normed[sel] = z
        z = rope_interleaved(z, np.asarray(cos)[sel], np.asarray(sin)[sel], int(rope_head_dim))
        if rotate:
            z = hadamard_rotate(z, a["hadamard"])
        out_f[sel] = z
    out = f64_to_bf16_bits(np.where(np.isnan(out_f), 0.0, out_f))

    kv_new = a["kv_state"].copy()
    sc_new = a["score_state"].copy()
    written = np.zeros(kv_new.shape[:2], dtype=bool)
    written_score = np.zeros(sc_new.shape[:2], dtype=bool)
    if write_state:
        for b in range(B):
            s, L = int(sp[b]), int(lay.length[b])
            e = s + L
            # Tail rule: keep exactly the rows a later call can still read. The
            # earliest window a later call completes is e // ratio; it reads
            # positions from (e // ratio - coff + 1) * ratio on.
            thr = (e // ratio - coff + 1) * ratio
            pos = np.arange(max(s, thr), e, dtype=np.int64)
            if pos.size == 0:
                continue
            kv, sc = seqs[b].current(pos) if seqs[b].kv is None else (
                seqs[b].kv[pos - s], seqs[b].sc[pos - s])
            r, o = seqs[b].slot(a["kv_block_table"], pos)
            kv_new[r, o] = kv
            written[r, o] = True
            r2, o2 = seqs[b].slot(a["state_block_table"], pos)
            sc_new[r2, o2] = sc
            written_score[r2, o2] = True
    return Result(out=out, out_f64=out_f, pooled=pooled, normed=normed,
                  kv_state=kv_new, score_state=sc_new, written=written,
                  written_score=written_score, layout=lay)


def run_inputs(inp, **kw) -> Result:
    """``compressor`` on a ``workloads.Inputs`` bundle."""
    return compressor(inp.x, inp.kv_state, inp.score_state, inp.kv_block_table,
                      inp.state_block_table, inp.sin, inp.cos, inp.wkv, inp.wgate, inp.ape,
                      inp.norm_weight, inp.hadamard, inp.start_pos, inp.cu_seqlens,
                      inp.ratio, inp.rope_head_dim, inp.rotate, **kw)


def window_row_positions(cu_seqlens, start_pos, ratio: int) -> np.ndarray:
    """RoPE position of each output row: window w sits at position w * ratio; rows
    with no window get position 0. (A convention for building sin/cos inputs.)"""
    lay = layout(cu_seqlens, start_pos, ratio)
    pos = np.zeros(lay.n_out, dtype=np.int64)
    for row, b, w in lay.rows:
        pos[row] = w * ratio
    return pos
