"""CPU oracle for NsaCompressWithCache (the NSA inference-time KV compression).

TEST INFRASTRUCTURE ONLY: the same rules as ``oracle.compressor`` apply (only
the tests, the smoke check and the benchmark's CPU leg may import it; it
shares no code with the CUDA library).

Source: "CANN ops-transformer 算子解析 NsaCompressWithCache 推理阶段 NSA KV 压缩
算子实战指南" — 功能说明与压缩算法流程 (the four steps), 计算公式, 参数说明,
约束说明, and the kernel description (values cast to fp32 before the multiply
and the reduction, one round-to-nearest-even cast back to fp16 / bf16).

What it computes, per batch b with s = act_seq_len[b] (lengths, type 1):

* trigger: s >= compress_block_size and (s - compress_block_size) % stride == 0;
  otherwise nothing is written for b;
* compress_idx = (s - compress_block_size) / stride; the tokens are positions
  compress_idx * stride .. + compress_block_size - 1, i.e. the last
  compress_block_size tokens of the batch;
* a token at position p is read from the paged cache [block_num,
  page_block_size, N, D] at (block_table[b][p // page_block_size],
  p % page_block_size), or, in the packed TND layout [T, N, D], at row
  sum(act_seq_len[:b]) + p;
* output_cache[slot_mapping[b], n, d] = round(sum_j input[token j, n, d] *
  weight[j, n]).

Arithmetic: the products and the sum are exact in float64 (at most 64 terms
of 16-bit values); the sum is rounded once to the cache dtype. The library
accumulates in fp32, so the comparison allows the fp32 accumulation error plus
one unit of the cache dtype.
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

from .compressor import bf16_to_f64, f64_to_bf16_bits


def half_to_f64(bits) -> np.ndarray:
    """fp16 bit patterns (uint16) -> exact float64 values."""
    return np.ascontiguousarray(np.asarray(bits, dtype=np.uint16)).view(np.float16).astype(np.float64)


def f64_to_half_bits(v) -> np.ndarray:
    """One round-to-nearest-even rounding of float64 values to fp16 (uint16 bits).
    numpy's float64 -> float16 conversion is a single IEEE rounding."""
    with np.errstate(over="ignore"):
        return np.asarray(v, dtype=np.float64).astype(np.float16).view(np.uint16)


def to_f64(bits, dtype: str) -> np.ndarray:
    return half_to_f64(bits) if dtype == "fp16" else bf16_to_f64(bits)


def to_bits(v, dtype: str) -> np.ndarray:
    return f64_to_half_bits(v) if dtype == "fp16" else f64_to_bf16_bits(v)


def triggers(s: int, compress_block_size: int, stride: int) -> bool:
    """The compression condition of 算法流程 step 1."""
    return s >= compress_block_size and (s - compress_block_size) % stride == 0


@dataclasses.dataclass
class NsaResult:
    output_cache: np.ndarray   # uint16 bits, the whole cache after the call
    written: np.ndarray        # bool [result_len]: slots this call wrote
    sums: np.ndarray           # float64 [result_len, N, D] exact sums (NaN where not written)
    abs_sums: np.ndarray       # float64 [result_len, N, D] exact sums of |product| (NaN where not
                               # written): the scale of any finite-precision summation's error


def nsa_compress(input_bits, weight_bits, slot_mapping, act_seq_len, block_table, output_cache_bits, *,
                 dtype: str, compress_block_size: int, compress_stride: int,
                 page_block_size: Optional[int] = None, layout: str = "paged") -> NsaResult:
    """One call. ``input_bits``: uint16 [block_num, page_block_size, N, D] (paged) or
    [T, N, D] (layout "TND"); ``weight_bits`` uint16 [compress_block_size, N];
    ``slot_mapping`` int [B]; ``act_seq_len`` int [B] (per-batch lengths);
    ``block_table`` int [B, blocks_per_batch] (paged only); ``output_cache_bits``
    uint16 [result_len, N, D] (not modified: the new cache is returned)."""
    if dtype not in ("fp16", "bf16"):
        raise ValueError("dtype is fp16 or bf16")
    inp = np.asarray(input_bits, dtype=np.uint16)   # converted token by token below
    w = to_f64(weight_bits, dtype)
    out = np.array(output_cache_bits, dtype=np.uint16, copy=True)
    result_len, N, D = out.shape
    cbs, stride = int(compress_block_size), int(compress_stride)
    if w.shape != (cbs, N):
        raise ValueError("weight must be [compress_block_size, N]")
    lens = np.asarray(act_seq_len, dtype=np.int64)
    slots = np.asarray(slot_mapping, dtype=np.int64)
    B = lens.shape[0]
    start = np.concatenate([[0], np.cumsum(lens)])  # TND row of each batch's first token
    written = np.zeros(result_len, dtype=bool)
    sums = np.full((result_len, N, D), np.nan)
    abs_sums = np.full((result_len, N, D), np.nan)
    for b in range(B):
        s = int(lens[b])
        if not triggers(s, cbs, stride):
            continue
        idx = (s - cbs) // stride
        acc = np.zeros((N, D))
        mag = np.zeros((N, D))
        for j in range(cbs):
            p = idx * stride + j
            if layout == "paged":
                blk = int(block_table[b][p // page_block_size])
                tok = inp[blk, p % page_block_size]
            else:
                tok = inp[int(start[b]) + p]
            prod = to_f64(tok, dtype) * w[j][:, None]
            acc += prod
            mag += np.abs(prod)
        slot = int(slots[b])
        out[slot] = to_bits(acc, dtype)
        sums[slot] = acc
        abs_sums[slot] = mag
        written[slot] = True
    return NsaResult(output_cache=out, written=written, sums=sums, abs_sums=abs_sums)


def nsa_compress_brute(input_bits, weight_bits, slot_mapping, act_seq_len, block_table,
                       output_cache_bits, *, dtype, compress_block_size, compress_stride,
                       page_block_size=None, layout="paged"):
    """The same definition with plain Python loops over every element (tiny inputs),
    written from the formula independently of ``nsa_compress``; returns the exact
    sums as {(slot, n, d): value}."""
    conv = (lambda bits: float(np.uint16(bits).view(np.float16))) if dtype == "fp16" else (
        lambda bits: float(np.array([int(bits) << 16], dtype=np.uint32).view(np.float32)[0]))
    res = {}
    B = len(act_seq_len)
    cbs, stride = int(compress_block_size), int(compress_stride)
    W = np.asarray(weight_bits)
    X = np.asarray(input_bits)
    N, D = np.asarray(output_cache_bits).shape[1:]
    for b in range(B):
        s = int(act_seq_len[b])
        if s < cbs or (s - cbs) % stride != 0:
            continue
        first = s - cbs  # (s - cbs) // stride * stride
        before = sum(int(act_seq_len[i]) for i in range(b))
        for n in range(N):
            for d in range(D):
                total = 0.0
                for j in range(cbs):
                    p = first + j
                    if layout == "paged":
                        blk = int(block_table[b][p // page_block_size])
                        v = conv(X[blk][p % page_block_size][n][d])
                    else:
                        v = conv(X[before + p][n][d])
                    total += v * conv(W[j][n])
                res[(int(slot_mapping[b]), n, d)] = total
    return res
