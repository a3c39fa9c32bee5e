"""Pure-Python brute force of the Compressor for tiny inputs.

TEST INFRASTRUCTURE ONLY: a second, independent statement of the same
computation, used to pin ``oracle.compressor``. It is written from the closed
form on "NPU DeepSeek-V4 Ascend C 融合算子优化" (Compressor 计算公式, C4A 层 and
C128A 层):

    C_i^Comp = sum_j exp(Z_j + B_j) * C_j  /  sum_j exp(Z_j + B_j)

with explicit Python loops and ``math`` only: no numpy, no softmax helper, no
max subtraction (inputs here are small, so exp cannot overflow). The
projections are dot products summed term by term and then rounded to float32
with ``struct`` (the state dtype); RMSNorm, RoPE and the Hadamard product are
loops over channels. Everything stays in Python floats (IEEE double).
"""

from __future__ import annotations

import math
import struct
from typing import Dict, List, Sequence, Tuple


def _bf16(u: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(u) & 0xFFFF) << 16))[0]


def _f32(v: float) -> float:
    return struct.unpack("<f", struct.pack("<f", v))[0]


def compress(x: Sequence[Sequence[int]], kv_state, score_state, kv_block_table,
             state_block_table, sin, cos, wkv, wgate, ape, norm_weight, hadamard,
             start_pos, cu_seqlens, ratio: int, rope_head_dim: int, rotate: bool):
    """Returns (windows, kv_state, score_state).

    ``windows`` maps (sequence, window index) -> list of D output floats before the
    bf16 rounding; ``sin``/``cos`` are looked up by the output row, which the caller
    supplies through ``row_of[(b, w)]`` in the tables' place: here sin/cos are dicts
    keyed by (b, w) giving the rope_head_dim-long bf16 rows.
    All array arguments are nested Python lists (bf16 tensors as uint16 ints).
    """
    coff = 2 if ratio == 4 else 1
    C = len(wkv)
    D = C // coff
    H = len(wkv[0])
    bs = len(kv_state[0])
    kv_new = [[list(r) for r in blk] for blk in kv_state]
    sc_new = [[list(r) for r in blk] for blk in score_state]
    B = len(cu_seqlens) - 1
    windows: Dict[Tuple[int, int], List[float]] = {}
    for b in range(B):
        s = 0 if start_pos is None else int(start_pos[b])
        t0, t1 = int(cu_seqlens[b]), int(cu_seqlens[b + 1])
        e = s + (t1 - t0)
        # rows of this call, by absolute position
        cur: Dict[int, Tuple[List[float], List[float]]] = {}
        for t in range(t0, t1):
            p = s + (t - t0)
            kv_row, sc_row = [], []
            for c in range(C):
                acc_k = 0.0
                acc_g = 0.0
                for h in range(H):
                    xv = _bf16(x[t][h])
                    acc_k += xv * _bf16(wkv[c][h])
                    acc_g += xv * _bf16(wgate[c][h])
                kv_row.append(_f32(acc_k))
                sc_row.append(_f32(acc_g + float(ape[p % ratio][c])))
            cur[p] = (kv_row, sc_row)

        def row(q):
            if q >= s:
                return cur[q]
            kb = kv_block_table[b][q // bs]
            sb = state_block_table[b][q // bs]
            return (list(kv_state[kb][q % bs]), list(score_state[sb][q % bs]))

        for p in range(s, e):
            if (p + 1) % ratio != 0:
                continue
            w = p // ratio
            y = []
            for c in range(D):
                num = 0.0
                den = 0.0
                if coff == 1:
                    for q in range(w * ratio, (w + 1) * ratio):
                        k_row, z_row = row(q)
                        g = math.exp(z_row[c])
                        num += g * k_row[c]
                        den += g
                else:
                    if w > 0:  # the first window has no previous one (weight 0)
                        for q in range((w - 1) * ratio, w * ratio):
                            k_row, z_row = row(q)
                            g = math.exp(z_row[c])
                            num += g * k_row[c]
                            den += g
                    for q in range(w * ratio, (w + 1) * ratio):
                        k_row, z_row = row(q)
                        g = math.exp(z_row[D + c])
                        num += g * k_row[D + c]
                        den += g
                y.append(num / den)
            ms = 0.0
            for c in range(D):
                ms += y[c] * y[c]
            inv = 1.0 / math.sqrt(ms / D + 1e-6)
            z = [y[c] * inv * _bf16(norm_weight[c]) for c in range(D)]
            cr = [_bf16(v) for v in cos[(b, w)]]
            sr = [_bf16(v) for v in sin[(b, w)]]
            half = rope_head_dim // 2
            base = D - rope_head_dim
            zr = list(z)
            for j in range(half):
                a0 = z[base + 2 * j]
                a1 = z[base + 2 * j + 1]
                zr[base + 2 * j] = a0 * cr[j] - a1 * sr[j]
                zr[base + 2 * j + 1] = a1 * cr[half + j] + a0 * sr[half + j]
            if rotate:
                o = []
                for jj in range(D):
                    acc = 0.0
                    for ii in range(D):
                        acc += zr[ii] * _bf16(hadamard[ii][jj])
                    o.append(acc)
                zr = o
            windows[(b, w)] = zr
        thr = (e // ratio - coff + 1) * ratio
        for p in range(s, e):
            if p < thr:
                continue
            kb = kv_block_table[b][p // bs]
            sb = state_block_table[b][p // bs]
            kv_new[kb][p % bs] = list(cur[p][0])
            sc_new[sb][p % bs] = list(cur[p][1])
    return windows, kv_new, sc_new
