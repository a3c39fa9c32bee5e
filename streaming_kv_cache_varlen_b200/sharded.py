"""One long prefill sharded by tokens across ranks (one process per GPU).

The Compressor's windows are independent once their rows are known, so a
single sequence of T tokens (positions 0 .. T-1) splits into window-aligned
token ranges, one per rank. No data crosses ranks before the end:

* ratio 128 (coff 1): rank k's windows use only its own tokens.
* ratio 4 (coff 2): the first window of rank k also needs the a-half of the
  previous window (the ratio tokens just before its range). The rank
  recomputes it from those tokens of x (a halo): its call starts ratio tokens
  early, so it also completes the previous rank's last window, whose row it
  drops. That row's own a-half would come from the paged state, which the
  rank backs with a zeroed scratch pool (the row is dropped anyway).

Each rank then holds the output rows of its windows; one all-gather of those
bf16 rows (about 1 MB for a 128K call) gives every rank the whole output. The
state tail of the sequence (the rows a later call would read) is produced by
the last rank, in its scratch state (the plan gives the last rank the last
window).

This is the context-parallel split of the pages' model integration ("compressor
torch_extension API", the CP all-gather of compressed rows), applied to the
Compressor alone. ``run_call`` is the per-rank compute (the CUDA library by
default); the gather uses torch.distributed (NCCL on GPUs, gloo on CPU).
"""

from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional


@dataclasses.dataclass(frozen=True)
class Shard:
    rank: int
    lo: int            # first token the rank owns (window aligned)
    hi: int            # one past its last token
    x_lo: int          # first token of its call: lo minus the halo
    first_window: int  # first window it emits
    n_windows: int     # windows it emits
    skip_rows: int     # leading output rows of its call that belong to the previous rank


def plan(T: int, ratio: int, world: int) -> List[Shard]:
    """Window-aligned token ranges for a sequence of T tokens from position 0.

    Windows are dealt out as evenly as possible, the spare ones to the last
    ranks, so that the last rank holds the last window whenever there is one; it
    also takes the tokens after the last complete window. The state tail (the
    rows from the last complete window on for ratio 4, the trailing tokens
    otherwise) therefore lies inside the last rank's call."""
    if T < 0 or ratio < 1 or world < 1:
        raise ValueError("T >= 0, ratio >= 1, world >= 1")
    coff = 2 if ratio == 4 else 1
    nwin = T // ratio
    base, extra = divmod(nwin, world)
    shards, w = [], 0
    for k in range(world):
        n = base + (1 if k >= world - extra else 0)
        lo, hi = w * ratio, (w + n) * ratio
        if k == world - 1:
            hi = T
        halo = (coff - 1) * ratio if (coff == 2 and w > 0 and hi > lo) else 0
        shards.append(Shard(k, lo, hi, lo - halo, w, n, 1 if halo else 0))
        w += n
    return shards


def n_out_rows(T: int, ratio: int) -> int:
    """Output rows of a one-sequence call: min(T, T // ratio + 1)."""
    return min(T, T // ratio + 1)


def local_layout(shard: Shard, ratio: int, block_size: int):
    """Positions, paged-state blocks and output rows of a shard's call.

    Returns (L, start_pos, n_out_local, block_lo, n_blocks, table_stride): the call
    covers tokens [x_lo, hi) at positions x_lo.., its state pool backs blocks
    block_lo .. block_lo + n_blocks - 1 (every block the call may read or write,
    including the previous window of its first window), and its output has
    n_out_local rows."""
    coff = 2 if ratio == 4 else 1
    L = shard.hi - shard.x_lo
    first_pos = max(0, shard.x_lo - (coff - 1) * ratio)
    block_lo = first_pos // block_size
    block_hi = max(shard.hi - 1, first_pos) // block_size
    return (L, shard.x_lo, min(L, L // ratio + 1), block_lo, block_hi - block_lo + 1, block_hi + 1)


def local_inputs(shard: Shard, x, sin, cos, ratio: int, block_size: int, C: int, device=None):
    """Tensors of a shard's call (torch): x slice, start_pos, cu_seqlens, one
    zeroed scratch pool for both states, its table, and sin / cos rows.

    ``x`` is the whole sequence [T, H] (or at least rows x_lo .. hi-1 at their
    positions); ``sin`` / ``cos`` are the whole call's tables [n_out, rope]."""
    import torch
    device = device if device is not None else x.device
    L, sp, n_loc, block_lo, n_blocks, stride = local_layout(shard, ratio, block_size)
    xs = x[shard.x_lo:shard.hi].contiguous()
    table = torch.full((1, stride), -1, dtype=torch.int32, device=device)
    table[0, block_lo:block_lo + n_blocks] = torch.arange(n_blocks, dtype=torch.int32, device=device)
    kv = torch.zeros((n_blocks, block_size, C), dtype=torch.float32, device=device)
    sc = torch.zeros_like(kv)
    rope = sin.shape[1]
    sin_l = torch.zeros((n_loc, rope), dtype=sin.dtype, device=device)
    cos_l = torch.zeros_like(sin_l)
    w0 = shard.x_lo // ratio  # window of local row 0
    nw_loc = min(n_loc, shard.n_windows + shard.skip_rows)
    if nw_loc > 0:
        sin_l[:nw_loc] = sin[w0:w0 + nw_loc]
        cos_l[:nw_loc] = cos[w0:w0 + nw_loc]
    return dict(x=xs, start_pos=torch.tensor([sp], dtype=torch.int32, device=device),
                cu_seqlens=torch.tensor([0, L], dtype=torch.int32, device=device),
                kv_state=kv, score_state=sc, kv_block_table=table, state_block_table=table.clone(),
                sin=sin_l, cos=cos_l)


def own_rows(shard: Shard, out_local):
    """The rows of a shard's call output that are its windows."""
    return out_local[shard.skip_rows:shard.skip_rows + shard.n_windows]


def assemble(shards: List[Shard], rows_per_rank, T: int, ratio: int, like):
    """Concatenate the ranks' rows in window order and append the zero rows a
    one-shot call has after its windows (``like``: a tensor of the right dtype
    and width)."""
    import torch
    n_out = n_out_rows(T, ratio)
    parts = [r for r in rows_per_rank]
    nwin = sum(s.n_windows for s in shards)
    out = torch.cat(parts, dim=0) if parts else like.new_zeros((0, like.shape[1]))
    if n_out > nwin:
        out = torch.cat([out, like.new_zeros((n_out - nwin, like.shape[1]))], dim=0)
    return out


def all_gather_rows(shards: List[Shard], mine, group=None):
    """Every rank's own rows, gathered in rank order (one all_gather of equal,
    padded blocks; pairs of 16-bit values travel as int32, which every backend
    carries, gloo included)."""
    import torch
    import torch.distributed as dist
    width = mine.shape[1]
    if width % 2:
        raise ValueError("row width must be even")
    cap = max(s.n_windows for s in shards)
    buf = torch.zeros((cap, width // 2), dtype=torch.int32, device=mine.device)
    if mine.shape[0]:
        buf[:mine.shape[0]] = mine.contiguous().view(torch.int32)
    bufs = [torch.empty_like(buf) for _ in shards]
    dist.all_gather(bufs, buf, group=group)
    return [b[:s.n_windows].view(mine.dtype) for b, s in zip(bufs, shards)]


def sharded_prefill(x, wkv, wgate, ape, norm_weight, hadamard, sin, cos, *, ratio: int,
                    rope_head_dim: int, rotate: bool, block_size: int, rank: int, world: int,
                    group=None, run_call: Optional[Callable] = None):
    """One sequence of T = x.shape[0] tokens from position 0, split across `world`
    ranks; returns (out [n_out, D] on every rank, this rank's call inputs — whose
    scratch states hold the sequence's tail on the last rank).

    ``run_call(**kwargs) -> out`` computes one Compressor call; by default the CUDA
    library (``streaming_kv_cache_varlen_b200.compressor``)."""
    if run_call is None:
        from . import compressor as run_call
    T = x.shape[0]
    C = wkv.shape[0]
    shards = plan(T, ratio, world)
    me = shards[rank]
    loc = local_inputs(me, x, sin, cos, ratio, block_size, C)
    out_loc = run_call(wkv=wkv, wgate=wgate, ape=ape, norm_weight=norm_weight, hadamard=hadamard,
                       ratio=ratio, rope_head_dim=rope_head_dim, rotate=rotate, **loc)
    mine = own_rows(me, out_loc)
    if world == 1:
        rows = [mine]
    else:
        rows = all_gather_rows(shards, mine, group=group)
    return assemble(shards, rows, T, ratio, mine), loc
