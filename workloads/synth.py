"""Seeded synthetic workloads for the Compressor.

Every array is drawn from one numpy PCG64 generator per workload, in a fixed
order, so the CPU oracle and the CUDA path see identical bytes. Tensors the
operator takes in bf16 are stored as uint16 bit patterns (numpy has no bf16).

Distribution notation: ``N(0, v)`` means mean 0 and *variance* v, so weights
drawn as ``N(0, 1/H)`` give projections of unit variance.

The five named workloads follow the Compressor pages' three typical layer
combinations (C4A: D=512, coff=2, ratio=4; C4Li: D=128, coff=2, ratio=4;
C128A: D=512, coff=1, ratio=128) and their streaming/varlen use: one-shot
prefill, packed varlen prefill, 128K prefill, 32-way decode and chunked
prefill continued over several calls with reordered requests.

Nothing here computes any part of the operator: the block tables only say
which pool row backs which ``block_size`` positions of each request, and the
RoPE tables are plain cos/sin of given positions.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

CONFIG_NAMES = ("c4li_tiny", "c4a_varlen", "c128a_128k", "c4a_decode", "c4li_chunked")


# ----------------------------------------------------------------------------
# dtype helpers (input creation only)
# ----------------------------------------------------------------------------

def bf16_bits(a) -> np.ndarray:
    """float32 values -> bf16 bit patterns (uint16), round to nearest even."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    rounding_bias = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding_bias) >> 16).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) -> exact float32 values."""
    b = np.ascontiguousarray(np.asarray(bits, dtype=np.uint16))
    return (b.astype(np.uint32) << 16).view(np.float32)


def sylvester(n: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix of order n (n a power of 2), int8 +-1."""
    if n < 1 or n & (n - 1):
        raise ValueError("order must be a power of two")
    h = np.ones((1, 1), dtype=np.int8)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def hadamard_bits(d: int) -> np.ndarray:
    """Sylvester H_d / sqrt(d) as bf16 bits, the rotation matrix the C4Li path takes."""
    return bf16_bits(sylvester(d).astype(np.float32) / np.float32(math.sqrt(d)))


def rope_tables(positions: Sequence[int], rope_dim: int = 64, base: float = 10000.0):
    """(cos, sin) bf16 bit tables of shape [len(positions), rope_dim].

    Column j and column rope_dim/2 + j both hold the angle pos * base**(-2j/rope_dim)
    (the half-duplicated layout of rotate-half RoPE tables).
    """
    pos = np.asarray(positions, dtype=np.float64).reshape(-1, 1)
    half = rope_dim // 2
    inv_freq = base ** (-(2.0 * np.arange(half, dtype=np.float64)) / rope_dim)
    ang = pos * inv_freq.reshape(1, -1)
    ang = np.concatenate([ang, ang], axis=1)
    return bf16_bits(np.cos(ang).astype(np.float32)), bf16_bits(np.sin(ang).astype(np.float32))


# ----------------------------------------------------------------------------
# container
# ----------------------------------------------------------------------------

@dataclasses.dataclass
class Inputs:
    name: str
    ratio: int
    coff: int
    D: int
    rope_head_dim: int
    rotate: bool
    block_size: int
    x: np.ndarray                 # uint16 [T, H]
    wkv: np.ndarray               # uint16 [coff*D, H]
    wgate: np.ndarray             # uint16 [coff*D, H]
    ape: np.ndarray               # float32 [ratio, coff*D]
    norm_weight: np.ndarray       # uint16 [D]
    hadamard: Optional[np.ndarray]  # uint16 [D, D] or None
    start_pos: np.ndarray         # int32 [B]
    cu_seqlens: np.ndarray        # int32 [B+1]
    kv_state: np.ndarray          # float32 [block_num, block_size, coff*D]
    score_state: np.ndarray       # float32 [block_num, block_size, coff*D]
    kv_block_table: np.ndarray    # int32 [B, table_stride]
    state_block_table: np.ndarray  # int32 [B, table_stride]
    sin: Optional[np.ndarray] = None  # uint16 [n_rows, rope_head_dim]
    cos: Optional[np.ndarray] = None

    @property
    def B(self) -> int:
        return int(self.cu_seqlens.shape[0] - 1)

    @property
    def T(self) -> int:
        return int(self.x.shape[0])

    @property
    def H(self) -> int:
        return int(self.x.shape[1])

    @property
    def C(self) -> int:
        return int(self.wkv.shape[0])

    @property
    def block_num(self) -> int:
        return int(self.kv_state.shape[0])

    @property
    def table_stride(self) -> int:
        return int(self.kv_block_table.shape[1])

    def with_rope(self, row_positions: Sequence[int], base: float = 10000.0) -> "Inputs":
        cos, sin = rope_tables(row_positions, self.rope_head_dim, base)
        return dataclasses.replace(self, cos=cos, sin=sin)


# ----------------------------------------------------------------------------
# generic builder
# ----------------------------------------------------------------------------

def _normal_bf16(rng: np.random.Generator, shape, var: float, mean: float = 0.0) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if var != 1.0:
        a *= np.float32(math.sqrt(var))
    if mean != 0.0:
        a += np.float32(mean)
    return bf16_bits(a)


def _block_lists(lengths, start_pos, block_size, lookback):
    """Per request, the block indices that get a pool row.

    lookback=None: every block from position 0 to the request's last position
    (a fully resident history). Otherwise only positions [start - lookback, end).
    """
    out = []
    for L, s in zip(lengths, start_pos):
        end = int(s) + int(L)
        lo = 0 if lookback is None else max(0, int(s) - int(lookback))
        if end <= lo:
            out.append([])
            continue
        out.append(list(range(lo // block_size, (end - 1) // block_size + 1)))
    return out


def _tables(rng, blocks, table_stride, extra_rows, separate_tables):
    n_used = sum(len(b) for b in blocks)
    block_num = n_used + extra_rows
    B = len(blocks)
    perm_kv = rng.permutation(block_num).astype(np.int32)
    perm_sc = rng.permutation(block_num).astype(np.int32) if separate_tables else perm_kv
    kv_t = np.full((B, table_stride), -1, dtype=np.int32)
    sc_t = np.full((B, table_stride), -1, dtype=np.int32)
    k = 0
    for b, bl in enumerate(blocks):
        for j in bl:
            kv_t[b, j] = perm_kv[k]
            sc_t[b, j] = perm_sc[k]
            k += 1
    return block_num, kv_t, sc_t


def make_inputs(*, name: str, seed: int, lengths: Sequence[int], start_pos: Sequence[int],
                H: int, D: int, coff: int, ratio: int, block_size: int, rotate: bool,
                rope_head_dim: int = 64, table_stride: Optional[int] = None,
                lookback: Optional[int] = None, extra_rows: int = 0,
                separate_tables: bool = False, x_var: float = 1.0,
                ape_var: float = 0.1, norm_var: float = 0.05, state_var: float = 1.0,
                rng: Optional[np.random.Generator] = None) -> Inputs:
    """Draw one workload. Order of draws: x, wkv, wgate, ape, norm_weight, state, tables."""
    rng = np.random.Generator(np.random.PCG64(seed)) if rng is None else rng
    lengths = [int(v) for v in lengths]
    start_pos = [int(v) for v in start_pos]
    B = len(lengths)
    T = sum(lengths)
    C = coff * D
    x = _normal_bf16(rng, (T, H), x_var)
    wkv = _normal_bf16(rng, (C, H), 1.0 / H)
    wgate = _normal_bf16(rng, (C, H), 1.0 / H)
    ape = (rng.standard_normal(size=(ratio, C), dtype=np.float32) * np.float32(math.sqrt(ape_var)))
    norm_weight = _normal_bf16(rng, (D,), norm_var, mean=1.0)
    hadamard = hadamard_bits(D) if rotate else None
    blocks = _block_lists(lengths, start_pos, block_size, lookback)
    if table_stride is None:
        table_stride = max([max(bl) + 1 for bl in blocks if bl] + [1])
    block_num = sum(len(b) for b in blocks) + extra_rows
    kv_state = rng.standard_normal(size=(block_num, block_size, C), dtype=np.float32)
    score_state = rng.standard_normal(size=(block_num, block_size, C), dtype=np.float32)
    if state_var != 1.0:
        kv_state *= np.float32(math.sqrt(state_var))
        score_state *= np.float32(math.sqrt(state_var))
    _, kv_t, sc_t = _tables(rng, blocks, table_stride, extra_rows, separate_tables)
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64)).astype(np.int32)
    return Inputs(name=name, ratio=ratio, coff=coff, D=D, rope_head_dim=rope_head_dim,
                  rotate=rotate, block_size=block_size, x=x, wkv=wkv, wgate=wgate, ape=ape,
                  norm_weight=norm_weight, hadamard=hadamard,
                  start_pos=np.asarray(start_pos, dtype=np.int32), cu_seqlens=cu,
                  kv_state=kv_state, score_state=score_state,
                  kv_block_table=kv_t, state_block_table=sc_t)


# ----------------------------------------------------------------------------
# the named workloads
# ----------------------------------------------------------------------------

def _decode_start_positions(rng, B, n_complete, ratio, lo, hi):
    """B positions uniform in [lo, hi); exactly n_complete of them are the last slot
    of a ratio-sized group (residue ratio-1), the rest have another residue."""
    which = np.zeros(B, dtype=bool)
    which[rng.choice(B, size=n_complete, replace=False)] = True
    out = []
    for b in range(B):
        while True:
            p = int(rng.integers(lo, hi))
            if (p % ratio == ratio - 1) == bool(which[b]):
                out.append(p)
                break
    return out


def make_config(name: str, seed: Optional[int] = None) -> Inputs:
    """One of the single-call workloads by name (the chunked one: ``make_chunked``)."""
    if name == "c4li_tiny":
        return make_inputs(name=name, seed=0 if seed is None else seed, lengths=[64],
                           start_pos=[0], H=1024, D=128, coff=2, ratio=4, block_size=16,
                           rotate=True, separate_tables=True, extra_rows=2)
    if name == "c4a_varlen":
        return make_inputs(name=name, seed=1 if seed is None else seed,
                           lengths=[1024, 3001, 5120, 7239], start_pos=[0, 0, 0, 0],
                           H=4096, D=512, coff=2, ratio=4, block_size=128, rotate=False)
    if name == "c128a_128k":
        return make_inputs(name=name, seed=2 if seed is None else seed, lengths=[131072],
                           start_pos=[0], H=4096, D=512, coff=1, ratio=128, block_size=128,
                           rotate=False)
    if name == "c4a_decode":
        rng = np.random.Generator(np.random.PCG64(3 if seed is None else seed))
        sp = _decode_start_positions(rng, 32, 8, 4, 4, 65536)
        return make_inputs(name=name, seed=0, rng=rng, lengths=[1] * 32, start_pos=sp,
                           H=4096, D=512, coff=2, ratio=4, block_size=128, rotate=False,
                           table_stride=512, lookback=8)
    raise KeyError(name)


@dataclasses.dataclass
class Chunked:
    """A chunked-prefill continuation: ``calls[i]`` is call i; ``order[i][j]`` is the
    request that sits in batch slot j of call i; ``oneshot`` is the whole sequences
    in one call (request j in slot j). The state arrays of ``calls[0]`` are the
    initial state; later calls carry the state their predecessor left."""
    calls: List[Inputs]
    order: List[np.ndarray]
    oneshot: Inputs
    chunk_lengths: np.ndarray   # [n_calls, B] by request


def make_chunked(seed: int = 4, *, B: int = 8, n_calls: int = 4, H: int = 7168, D: int = 128,
                 max_chunk: int = 2048, block_size: int = 128, rotate: bool = True,
                 ratio: int = 4, coff: int = 2) -> Chunked:
    rng = np.random.Generator(np.random.PCG64(seed))
    chunks = rng.integers(1, max_chunk + 1, size=(n_calls, B))
    total = chunks.sum(axis=0)
    oneshot = make_inputs(name="c4li_chunked_oneshot", seed=0, rng=rng,
                          lengths=total.tolist(), start_pos=[0] * B, H=H, D=D, coff=coff,
                          ratio=ratio, block_size=block_size, rotate=rotate)
    # per-request token rows inside the one-shot packing
    starts = oneshot.cu_seqlens[:-1].astype(np.int64)
    calls, orders = [], []
    done = np.zeros(B, dtype=np.int64)
    for c in range(n_calls):
        order = rng.permutation(B)
        lengths = [int(chunks[c, r]) for r in order]
        sp = [int(done[r]) for r in order]
        rows = np.concatenate([np.arange(starts[r] + done[r], starts[r] + done[r] + chunks[c, r])
                               for r in order])
        cu = np.zeros(B + 1, dtype=np.int32)
        cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64)).astype(np.int32)
        calls.append(dataclasses.replace(
            oneshot, name=f"c4li_chunked_call{c}", x=oneshot.x[rows],
            start_pos=np.asarray(sp, dtype=np.int32), cu_seqlens=cu,
            kv_block_table=oneshot.kv_block_table[order].copy(),
            state_block_table=oneshot.state_block_table[order].copy()))
        orders.append(order)
        done += chunks[c]
    return Chunked(calls=calls, order=orders, oneshot=oneshot, chunk_lengths=chunks)
