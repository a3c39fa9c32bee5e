"""Python binding of the B200 streaming KV-cache Compressor library.

A thin ctypes layer over the C ABI in include/cmp.h: it checks dtypes, devices
and shapes of PyTorch tensors, derives the shape scalars and passes raw
pointers. Every step of the computation runs in the library's CUDA kernels;
there is no other implementation behind these functions. Importing this
package fails if the library has not been built.
"""

from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
# CMP_LIBRARY selects another build of the same library (the phase-stamp
# measurement build libcmp_b200_phases.so); by default the one next to this file
LIB_PATH = os.environ.get("CMP_LIBRARY") or os.path.join(_PKG, "libcmp_b200.so")

CMP_OK = 0
STATUS = {0: "CMP_OK", 1: "CMP_ERR_NULLPTR", 2: "CMP_ERR_INVALID", 3: "CMP_ERR_UNSUPPORTED",
          4: "CMP_ERR_CUDA", 5: "CMP_ERR_DEVICE_INDEX", 6: "CMP_ERR_TIMEOUT"}
KERNELS = ("sched", "proj_tcgen05", "proj_mma_sync", "proj_decode", "pool_epilogue",
           "fused_tcgen05", "finish", "decode_fused", "decode_cp", "nsa_compress", "nsa_scan")


class CmpError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)}" if what else STATUS.get(status, str(status)))


class cmp_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("T", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("block_num", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("table_stride", ctypes.c_int32)]


class cmp_nsa_dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("N", ctypes.c_int64), ("D", ctypes.c_int64),
                ("tokens", ctypes.c_int64), ("table_stride", ctypes.c_int64),
                ("result_len", ctypes.c_int64)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -c 'import __graft_entry__ as g; g.build()'`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "cmp_out_rows": (I64, [I64, I64, I32]),
        "cmp_out_row_layout": (ctypes.c_int, [P, P, I32, I32, I64, P, P]),
        "cmp_compressor": (ctypes.c_int, [P] * 14 + [I32, I32, ctypes.c_bool, P, P,
                                                   ctypes.POINTER(cmp_dims)]),
        "cmp_compressor_noalloc": (ctypes.c_int, [P] * 14 + [I32, I32, ctypes.c_bool, P, P,
                                                           ctypes.POINTER(cmp_dims)]),
        "cmp_get_error": (ctypes.c_int, [P]),
        "cmp_debug_phase_stamps": (ctypes.c_int, [P, I64]),
        "cmp_workspace_size": (SZ, [ctypes.POINTER(cmp_dims), I32]),
        "cmp_release_workspaces": (ctypes.c_int, []),
        "cmp_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "cmp_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
        "cmp_launch_count": (I64, []),
        "cmp_profile_start": (ctypes.c_int, []),
        "cmp_profile_stop": (ctypes.c_int, [P, P]),
        "cmp_set_proj_kernel": (ctypes.c_int, [ctypes.c_int]),
        "cmp_debug_unreachable_barrier": (ctypes.c_int, [ctypes.c_int]),
        "cmp_nsa_compress": (ctypes.c_int, [P, P, P, P, P, I32, I32, I64, I64, I64, P, P,
                                            ctypes.POINTER(cmp_nsa_dims)]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


lib = _load()


def out_rows(B: int, T: int, ratio: int) -> int:
    """Rows of out / sin / cos: min(T, T // ratio + B)."""
    return int(lib.cmp_out_rows(B, T, ratio))


def out_row_layout(cu_seqlens, start_pos, ratio: int):
    """(row_seq, row_window) int32 numpy arrays of every output row (-1 = empty row)."""
    import numpy as np
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    B = cu.shape[0] - 1
    sp = None if start_pos is None else np.ascontiguousarray(np.asarray(start_pos, dtype=np.int32))
    n = out_rows(B, int(cu[-1]), ratio)
    rs = np.empty(max(n, 0), dtype=np.int32)
    rw = np.empty(max(n, 0), dtype=np.int32)
    st = lib.cmp_out_row_layout(cu.ctypes.data, None if sp is None else sp.ctypes.data, B, ratio, n,
                                rs.ctypes.data, rw.ctypes.data)
    if st != CMP_OK:
        raise CmpError(st, "cmp_out_row_layout")
    return rs, rw


def _ptr(t) -> Optional[int]:
    return None if t is None else int(t.data_ptr())


def _check(t, name, dtype, dim, device):
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def compressor(x, kv_state, score_state, kv_block_table, state_block_table, sin, cos, wkv, wgate,
               ape, norm_weight, hadamard, start_pos, cu_seqlens, ratio: int, rope_head_dim: int,
               rotate: bool, out=None, stream=None):
    """One Compressor call (see cmp_compressor in include/cmp.h); returns ``out``.

    x bf16 [T, H]; kv_state / score_state fp32 [block_num, block_size, coff*D] (updated
    in place); tables int32 [B, stride]; sin / cos bf16 [n_out, rope_head_dim]; wkv /
    wgate bf16 [coff*D, H]; ape fp32 [ratio, coff*D]; norm_weight bf16 [D]; hadamard bf16
    [D, D] or None; start_pos int32 [B] or None; cu_seqlens int32 [B+1]. All on one CUDA
    device. ``stream``: a torch.cuda.Stream or raw handle (default: current stream).
    """
    import torch
    dev = x.device
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    _check(x, "x", bf, 2, dev)
    _check(kv_state, "kv_state", f32, 3, dev)
    _check(score_state, "score_state", f32, 3, dev)
    _check(kv_block_table, "kv_block_table", i32, 2, dev)
    _check(state_block_table, "state_block_table", i32, 2, dev)
    _check(wkv, "wkv", bf, 2, dev)
    _check(wgate, "wgate", bf, 2, dev)
    _check(ape, "ape", f32, 2, dev)
    _check(norm_weight, "norm_weight", bf, 1, dev)
    _check(cu_seqlens, "cu_seqlens", i32, 1, dev)
    _check(sin, "sin", bf, 2, dev)
    _check(cos, "cos", bf, 2, dev)
    if hadamard is not None:
        _check(hadamard, "hadamard", bf, 2, dev)
    if start_pos is not None:
        _check(start_pos, "start_pos", i32, 1, dev)
    T, H = x.shape
    B = cu_seqlens.shape[0] - 1
    D = norm_weight.shape[0]
    C = wkv.shape[0]
    coff = 2 if ratio == 4 else 1
    n_out = out_rows(B, T, ratio)
    if C != coff * D or tuple(wgate.shape) != (C, H) or wkv.shape[1] != H:
        raise ValueError("wkv / wgate must be [coff*D, H] with D = norm_weight.numel()")
    if tuple(ape.shape) != (ratio, C):
        raise ValueError("ape must be [ratio, coff*D]")
    if kv_state.shape[2] != C or kv_state.shape != score_state.shape:
        raise ValueError("kv_state / score_state must both be [block_num, block_size, coff*D]")
    if kv_block_table.shape != state_block_table.shape or kv_block_table.shape[0] != B:
        raise ValueError("block tables must both be [B, table_stride]")
    if n_out > 0 and (tuple(sin.shape) != (n_out, rope_head_dim) or sin.shape != cos.shape):
        raise ValueError(f"sin / cos must be [{n_out}, {rope_head_dim}]")
    if start_pos is not None and start_pos.shape[0] != B:
        raise ValueError("start_pos must be [B]")
    if out is None:
        out = torch.empty((max(n_out, 0), D), dtype=bf, device=dev)
    else:
        _check(out, "out", bf, 2, dev)
        if tuple(out.shape) != (n_out, D):
            raise ValueError(f"out must be [{n_out}, {D}]")
    dims = cmp_dims(B, T, H, D, kv_state.shape[0], kv_state.shape[1], kv_block_table.shape[1])
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(dev):
        st = lib.cmp_compressor(_ptr(x), _ptr(kv_state), _ptr(score_state), _ptr(kv_block_table),
                                _ptr(state_block_table), _ptr(sin), _ptr(cos), _ptr(wkv),
                                _ptr(wgate), _ptr(ape), _ptr(norm_weight), _ptr(hadamard),
                                _ptr(start_pos), _ptr(cu_seqlens), ratio, rope_head_dim,
                                bool(rotate), _ptr(out), handle, ctypes.byref(dims))
    if st != CMP_OK:
        raise CmpError(st, "cmp_compressor")
    return out


def nsa_compress(input, weight, slot_mapping, act_seq_len, output_cache, *, compress_block_size: int,
                 compress_stride: int, block_table=None, page_block_size: int = 128, stream=None):
    """NsaCompressWithCache (see cmp_nsa_compress in include/cmp.h); updates and returns
    ``output_cache``.

    input fp16 / bf16: paged [block_num, page_block_size, N, D] (with ``block_table`` int32
    [B, pages per batch]) or packed [T, N, D]; weight [compress_block_size, N]; slot_mapping
    int32 [B]; act_seq_len int64 [B]; output_cache [result_len, N, D]. One CUDA device."""
    import torch
    dev = input.device
    if dev.type != "cuda":
        raise ValueError("tensors must be on a CUDA device")
    if input.dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("input must be float16 or bfloat16")
    paged = input.dim() == 4
    if not paged and input.dim() != 3:
        raise ValueError("input must be [block_num, page_block_size, N, D] or [T, N, D]")
    _check(input, "input", input.dtype, input.dim(), dev)
    _check(weight, "weight", input.dtype, 2, dev)
    _check(output_cache, "output_cache", input.dtype, 3, dev)
    _check(slot_mapping, "slot_mapping", torch.int32, 1, dev)
    _check(act_seq_len, "act_seq_len", torch.int64, 1, dev)
    result_len, N, D = output_cache.shape
    if tuple(input.shape[-2:]) != (N, D):
        raise ValueError("input and output_cache must share [N, D]")
    if tuple(weight.shape) != (compress_block_size, N):
        raise ValueError("weight must be [compress_block_size, N]")
    B = slot_mapping.shape[0]
    if act_seq_len.shape[0] != B:
        raise ValueError("act_seq_len must be [B]")
    if paged:
        if block_table is None:
            raise ValueError("the paged layout needs block_table")
        _check(block_table, "block_table", torch.int32, 2, dev)
        if block_table.shape[0] != B or input.shape[1] != page_block_size:
            raise ValueError("block_table must be [B, pages]; input [block_num, page_block_size, N, D]")
        tokens, stride = input.shape[0], block_table.shape[1]
    else:
        tokens, stride = input.shape[0], 1
    dims = cmp_nsa_dims(B, N, D, tokens, stride, result_len)
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(dev):
        st = lib.cmp_nsa_compress(_ptr(input), _ptr(weight), _ptr(slot_mapping), _ptr(act_seq_len),
                                  _ptr(block_table) if paged else None, 0 if paged else 1,
                                  1 if input.dtype == torch.bfloat16 else 0, compress_block_size,
                                  compress_stride, page_block_size if paged else 0,
                                  _ptr(output_cache), handle, ctypes.byref(dims))
    if st != CMP_OK:
        raise CmpError(st, "cmp_nsa_compress")
    return output_cache


def debug_check_tables(kv_block_table, state_block_table, cu_seqlens, start_pos, ratio: int,
                       block_size: int, block_num: int):
    """Host-side check of a call's documented preconditions, for tests and
    debugging (the library never runs it): every table entry the call reads or
    writes lies in [0, block_num), and no pool row is used by two sequences.
    Sequence b at positions [s, e) reads the rows before s of the windows it
    completes, from ((s // ratio) - coff + 1) * ratio on, only if it completes
    one; it writes its tail rows, from ((e // ratio) - coff + 1) * ratio on. Arguments are host arrays (numpy or CPU
    tensors). Returns a list of problems, empty when there are none."""
    import numpy as np

    def host(a):
        return None if a is None else np.asarray(a.cpu() if hasattr(a, "cpu") else a)

    kv, sc, cu = host(kv_block_table), host(state_block_table), host(cu_seqlens).astype(np.int64)
    B = cu.shape[0] - 1
    sp = np.zeros(B, dtype=np.int64) if start_pos is None else host(start_pos).astype(np.int64)
    coff = 2 if ratio == 4 else 1
    problems, owner = [], ({}, {})
    for b in range(B):
        s, e = int(sp[b]), int(sp[b]) + int(cu[b + 1] - cu[b])
        if e == s:
            continue
        blocks = set()
        w0 = s // ratio  # the first window the call can complete
        if (w0 + 1) * ratio <= e:  # it does: its rows before s come from the state
            read_lo = max(0, (w0 - coff + 1) * ratio)
            if read_lo < s:
                blocks.update(range(read_lo // block_size, (s - 1) // block_size + 1))
        write_lo = max(s, (e // ratio - coff + 1) * ratio)  # the tail rows
        if write_lo < e:
            blocks.update(range(write_lo // block_size, (e - 1) // block_size + 1))
        for which, table in enumerate((kv, sc)):
            for blk in sorted(blocks):
                if blk >= table.shape[1]:
                    problems.append(f"sequence {b}: block {blk} is past the table's {table.shape[1]} columns")
                    continue
                row = int(table[b, blk])
                if not 0 <= row < block_num:
                    problems.append(f"sequence {b}: table entry [{b}][{blk}] = {row} is outside [0, {block_num})")
                    continue
                other = owner[which].setdefault(row, b)
                if other != b:
                    name = "kv" if which == 0 else "score"
                    problems.append(f"{name} pool row {row} is used by sequences {other} and {b}")
    return problems


def get_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return int(lib.cmp_get_error(handle))


def workspace_size(B, T, H, D, block_num, block_size, table_stride, ratio) -> int:
    d = cmp_dims(B, T, H, D, block_num, block_size, table_stride)
    return int(lib.cmp_workspace_size(ctypes.byref(d), ratio))


def release_workspaces() -> None:
    st = lib.cmp_release_workspaces()
    if st != CMP_OK:
        raise CmpError(st, "cmp_release_workspaces")


def launch_count() -> int:
    return int(lib.cmp_launch_count())


def profile_start() -> None:
    lib.cmp_profile_start()


def profile_stop() -> Dict[str, Tuple[float, int]]:
    """{kernel name: (total ms, launches)} since profile_start()."""
    ms = (ctypes.c_double * len(KERNELS))()
    n = (ctypes.c_int64 * len(KERNELS))()
    st = lib.cmp_profile_stop(ms, n)
    if st != CMP_OK:
        raise CmpError(st, "cmp_profile_stop")
    return {KERNELS[i]: (float(ms[i]), int(n[i])) for i in range(len(KERNELS))}


def debug_unreachable_barrier(launches: int) -> int:
    """Testing knob: the next ``launches`` channel-group decode launches time out
    at their grid barrier (about 1 s each; get_error then reports
    CMP_ERR_TIMEOUT). Returns the previous count."""
    return int(lib.cmp_debug_unreachable_barrier(launches))


def set_proj_kernel(which: int) -> int:
    """Testing knob, which path calls take: 0 automatic, 1 mma.sync projection,
    2 tcgen05 projection (on CTA pairs where the device co-schedules them), 3 weight
    streaming, 4 fused tcgen05 pooling (on CTA pairs when the channel blocks pair up),
    5 K-split one-kernel decode, 6 channel-group one-kernel decode, 7 tcgen05
    projection on single CTAs, 8 fused path on single CTAs. Returns the previous value."""
    return int(lib.cmp_set_proj_kernel(which))


def debug_phase_stamps(n_ctas: int):
    """The channel-group decode kernel's phase stamps of its last launch, as a
    numpy uint64 array [n_ctas, 32] (global timer, ns). Only the phase-stamp
    measurement build (CMP_LIBRARY=.../libcmp_b200_phases.so) records them;
    other builds raise CmpError(CMP_ERR_UNSUPPORTED)."""
    import numpy as np
    buf = np.zeros((n_ctas, 32), dtype=np.uint64)
    st = lib.cmp_debug_phase_stamps(buf.ctypes.data, buf.size)
    if st != CMP_OK:
        raise CmpError(st, "cmp_debug_phase_stamps")
    return buf
