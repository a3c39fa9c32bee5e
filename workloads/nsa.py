"""Seeded synthetic inputs for NsaCompressWithCache.

One numpy PCG64 generator per workload, drawing in a fixed order: lengths,
cache, weight, block table, slot mapping, initial output cache. 16-bit values
are stored as uint16 bit patterns (fp16 through numpy's float16, bf16 through
``bf16_bits``). Nothing here computes any part of the operator.

Shapes follow the pages' example and constraints ("CANN ops-transformer 算子解析
NsaCompressWithCache": input [block_num, page_block_size, N, D] or [T, N, D],
weight [compress_block_size, N], slot_mapping [B], act_seq_len [B], block_table
[B, blocks_per_batch], output cache [result_len, N, D]).
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

from .synth import bf16_bits


@dataclasses.dataclass
class NsaInputs:
    name: str
    dtype: str                  # "fp16" or "bf16"
    layout: str                 # "paged" or "TND"
    compress_block_size: int
    compress_stride: int
    page_block_size: int
    input: np.ndarray           # uint16 [block_num, page_block_size, N, D] or [T, N, D]
    weight: np.ndarray          # uint16 [compress_block_size, N]
    slot_mapping: np.ndarray    # int32 [B]
    act_seq_len: np.ndarray     # int64 [B]
    block_table: np.ndarray     # int32 [B, blocks_per_batch] (paged; a dummy [B, 1] for TND)
    output_cache: np.ndarray    # uint16 [result_len, N, D], the cache before the call


def _bits(rng, shape, dtype, scale=1.0):
    v = rng.standard_normal(size=shape, dtype=np.float32) * np.float32(scale)
    return v.astype(np.float16).view(np.uint16) if dtype == "fp16" else bf16_bits(v)


def make_nsa_inputs(*, name: str, seed: int, B: int, N: int, D: int, compress_block_size: int,
                    compress_stride: int, page_block_size: int = 128, dtype: str = "bf16",
                    layout: str = "paged", lengths: Optional[Sequence[int]] = None,
                    max_seq_len: int = 512, result_len: Optional[int] = None,
                    trigger_fraction: float = 0.5, spare_blocks: int = 1) -> NsaInputs:
    """Batch lengths: given, or drawn in [compress_block_size, max_seq_len) with about
    ``trigger_fraction`` of them on a compression step (length - cbs a multiple of
    the stride). Paged: every batch owns ceil(max_seq_len / page_block_size) pool
    blocks, drawn from a random permutation (plus ``spare_blocks`` unused ones).
    Slots: a random injection of the batches into [0, result_len)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    cbs, stride = compress_block_size, compress_stride
    if lengths is None:
        lens = []
        for _ in range(B):
            if rng.random() < trigger_fraction:
                k = int(rng.integers(0, (max_seq_len - cbs) // stride + 1))
                lens.append(cbs + k * stride)
            else:
                lens.append(int(rng.integers(0, max_seq_len + 1)))
        lens = np.asarray(lens, dtype=np.int64)
    else:
        lens = np.asarray(lengths, dtype=np.int64)
        B = lens.shape[0]
    per = -(-max(max_seq_len, int(lens.max(initial=0))) // page_block_size)
    if layout == "paged":
        block_num = B * per + spare_blocks
        inp = _bits(rng, (block_num, page_block_size, N, D), dtype)
    else:
        inp = _bits(rng, (int(lens.sum()), N, D), dtype)
    weight = _bits(rng, (cbs, N), dtype, scale=1.0 / np.sqrt(cbs))
    if layout == "paged":
        perm = rng.permutation(block_num).astype(np.int32)
        table = perm[:B * per].reshape(B, per)
    else:
        table = np.zeros((B, 1), dtype=np.int32)
    if result_len is None:
        result_len = max(B, 1) * 2
    slots = rng.permutation(result_len)[:B].astype(np.int32)
    out0 = _bits(rng, (result_len, N, D), dtype)
    return NsaInputs(name=name, dtype=dtype, layout=layout, compress_block_size=cbs,
                     compress_stride=stride, page_block_size=page_block_size, input=inp,
                     weight=weight, slot_mapping=slots, act_seq_len=lens, block_table=table,
                     output_cache=out0)
