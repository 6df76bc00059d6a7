"""Thin ctypes binding of libspa.so (include/spa.h), with the same names.

Argument marshalling only: every step runs in the CUDA kernels behind the C-ABI.
PyTorch is used for device memory and the current stream. There is no CPU path:
importing this module without a built libspa.so raises, and every call needs CUDA
tensors.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

__all__ = ["SpaError", "lib", "spa_block_stats", "spa_select", "spa_sparse_attn_prefill",
           "spa_decode_workspace_bytes", "spa_sparse_attn_decode", "spa_get_device_error",
           "spa_status_string", "spa_last_error", "prefill", "decode", "LIB_PATH",
           "spa_prefill_host", "spa_prefill_host_workspace_bytes", "spa_selftest_wait_timeout"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libspa.so")

SPA_F32, SPA_BF16 = 0, 1
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_lib = None


class SpaError(RuntimeError):
    """A libspa call returned a non-zero spa_status."""

    def __init__(self, fn: str, status: int, detail: str):
        self.status = status
        super().__init__(f"{fn}: {_status_name(status)} (status {status}): {detail}")


def lib() -> ctypes.CDLL:
    """The loaded libspa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libspa.so not found at {LIB_PATH}; build it with "
                              "`python -m block_sparse_long_stats_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.spa_block_stats.argtypes = [_P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P]
        L.spa_select.argtypes = [_P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _I, _I, _I,
                                 _P, _I, _P, _P]
        L.spa_sparse_attn_prefill.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P,
                                              _F, _P, _P, _P]
        L.spa_decode_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
        L.spa_decode_workspace_bytes.restype = ctypes.c_size_t
        L.spa_sparse_attn_decode.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P,
                                             _F, _P, _P, _P]
        L.spa_rla_block_states.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P]
        L.spa_rla_prefill.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P, _P,
                                      _P]
        L.spa_rla_decode_state.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P]
        L.spa_rla_decode_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
        L.spa_rla_decode_workspace_bytes.restype = ctypes.c_size_t
        L.spa_sparse_attn_decode_rla.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P,
                                                 _I, _P, _F, _P, _P, _P, _P]
        L.spa_quantized_stats_bytes.argtypes = [_I, _I, _I, _I, _I]
        L.spa_quantized_stats_bytes.restype = ctypes.c_size_t
        L.spa_quantize_block_stats.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P]
        L.spa_block_stats_quantized.argtypes = [_P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _I, _P]
        L.spa_select_quantized.argtypes = [_P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _F, _I, _I,
                                           _I, _P, _I, _P, _P]
        L.spa_select_score_order.argtypes = [_P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _F, _F, _I,
                                             _I, _I, _P, _I, _P, _P]
        L.spa_sparse_attn_prefill_early_stop.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I,
                                                         _P, _I, _P, _F, _I, _I, _F, _P, _P, _P,
                                                         _P]
        L.spa_pbs_workspace_bytes.argtypes = [_I, _I, _I, _I, _I]
        L.spa_pbs_workspace_bytes.restype = ctypes.c_size_t
        L.spa_pbs_permutation.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _F, _P,
                                          ctypes.c_size_t, _P, _P]
        L.spa_pbs_gather.argtypes = [_P, _I, _I, _I, _I, _I, _P, _P, _P]
        L.spa_select_segperm.argtypes = [_P, _I, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F,
                                         _F, _I, _I, _I, _P, _I, _P, _P]
        L.spa_sparse_attn_prefill_segperm.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I,
                                                      _I, _I, _P, _I, _P, _F, _P, _P, _P]
        L.spa_prefill_host_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I, _I]
        L.spa_prefill_host_workspace_bytes.restype = ctypes.c_size_t
        L.spa_prefill_host.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _F, _I, _I,
                                       _I, _P, ctypes.c_size_t, _P]
        L.spa_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_int)]
        L.spa_selftest_wait_timeout.argtypes = [_I, _P]
        L.spa_status_string.argtypes = [_I]
        L.spa_status_string.restype = ctypes.c_char_p
        L.spa_last_error.restype = ctypes.c_char_p
        for f in ("spa_block_stats", "spa_select", "spa_sparse_attn_prefill",
                  "spa_sparse_attn_decode", "spa_get_device_error", "spa_rla_block_states",
                  "spa_rla_prefill", "spa_rla_decode_state", "spa_sparse_attn_decode_rla",
                  "spa_quantize_block_stats", "spa_select_quantized", "spa_select_score_order",
                  "spa_block_stats_quantized",
                  "spa_sparse_attn_prefill_early_stop", "spa_pbs_permutation", "spa_pbs_gather",
                  "spa_select_segperm", "spa_sparse_attn_prefill_segperm", "spa_prefill_host",
                  "spa_selftest_wait_timeout"):
            getattr(L, f).restype = _I
        _lib = L
    return _lib


def _status_name(st: int) -> str:
    return lib().spa_status_string(st).decode()


def spa_status_string(status: int) -> str:
    return _status_name(status)


def spa_last_error() -> str:
    return lib().spa_last_error().decode()


def _check(fn: str, st: int):
    if st != 0:
        raise SpaError(fn, st, spa_last_error())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libspa works on CUDA tensors only")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


_QFMT = {"int4": 0, "fp4": 1}


def _qfmt(fmt: str) -> int:
    if fmt not in _QFMT:
        raise ValueError(f"unknown record format {fmt!r} (int4 or fp4)")
    return _QFMT[fmt]


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SPA_BF16
    if t.dtype == torch.float32:
        return SPA_F32
    raise ValueError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def spa_block_stats(k: torch.Tensor, block: int, blk_begin: int = 0, blk_end: int | None = None,
                    mean: torch.Tensor | None = None, var: torch.Tensor | None = None,
                    stream=None):
    """Per-block key mean and variance: k [B,Hkv,T,d] -> mean, var [B,Hkv,nb,d] fp32."""
    B, Hkv, T, d = k.shape
    nb = -(-T // block)
    blk_end = nb if blk_end is None else blk_end
    if mean is None:
        mean = torch.empty((B, Hkv, nb, d), device=k.device, dtype=torch.float32)
    if var is None:
        var = torch.empty((B, Hkv, nb, d), device=k.device, dtype=torch.float32)
    _check("spa_block_stats", lib().spa_block_stats(_ptr(k), _dt(k), B, Hkv, T, d, block,
                                                    blk_begin, blk_end, _ptr(mean), _ptr(var),
                                                    _stream(stream)))
    return mean, var


def spa_select(q: torch.Tensor, mean: torch.Tensor, var: torch.Tensor, T: int, block: int,
               scale: float, top_p: float, n_sink: int = 1, n_local: int = 1, k_min: int = 0,
               idx: torch.Tensor | None = None, count: torch.Tensor | None = None,
               cap: int | None = None, stream=None):
    """Kept-block lists: q [B,Hq,Lq,d] (Lq = T or 1) -> idx [B,Hq,nq,cap], count [B,Hq,nq]."""
    B, Hq, Lq, d = q.shape
    Hkv = mean.shape[1]
    nb = -(-T // block)
    nq = -(-Lq // block)
    if idx is None:
        cap = nb if cap is None else cap
        idx = torch.empty((B, Hq, nq, cap), device=q.device, dtype=torch.int32)
    cap = idx.shape[-1]
    if count is None:
        count = torch.empty((B, Hq, nq), device=q.device, dtype=torch.int32)
    _check("spa_select", lib().spa_select(_ptr(q), _dt(q), _ptr(mean), _ptr(var), B, Hq, Hkv, Lq, T,
                                          d, block, scale, top_p, n_sink, n_local, k_min,
                                          _ptr(idx), cap, _ptr(count), _stream(stream)))
    return idx, count


def spa_quantized_stats_bytes(B: int, Hkv: int, T: int, d: int, block: int) -> int:
    return int(lib().spa_quantized_stats_bytes(B, Hkv, T, d, block))


def spa_quantize_block_stats(mean: torch.Tensor, var: torch.Tensor, T: int, block: int,
                             blk_begin: int = 0, blk_end: int | None = None,
                             qstats: torch.Tensor | None = None, fmt: str = "int4",
                             stream=None) -> torch.Tensor:
    """Microscale records [B, Hkv, nb, d + d/16] uint8 (fmt "int4" or "fp4") from fp32
    block statistics."""
    B, Hkv, nb, d = mean.shape
    if blk_end is None:
        blk_end = nb
    if qstats is None:
        qstats = torch.empty((B, Hkv, nb, d + d // 16), device=mean.device, dtype=torch.uint8)
    _check("spa_quantize_block_stats",
           lib().spa_quantize_block_stats(_ptr(mean), _ptr(var), B, Hkv, T, d, block, blk_begin,
                                          blk_end, _ptr(qstats), _qfmt(fmt), _stream(stream)))
    return qstats


def spa_block_stats_quantized(k: torch.Tensor, block: int, blk_begin: int, blk_end: int,
                              mean: torch.Tensor, var: torch.Tensor, qstats: torch.Tensor,
                              fmt: str = "int4", stream=None) -> None:
    """Statistics and records (fmt "int4" or "fp4") of blocks [blk_begin, blk_end) in
    one pass, into the caller's mean, var [B, Hkv, nb, d] and qstats [B, Hkv, nb,
    d + d/16]."""
    B, Hkv, T, d = k.shape
    _check("spa_block_stats_quantized",
           lib().spa_block_stats_quantized(_ptr(k), _dt(k), B, Hkv, T, d, block, blk_begin, blk_end,
                                           _ptr(mean), _ptr(var), _ptr(qstats), _qfmt(fmt),
                                           _stream(stream)))


def spa_select_quantized(q: torch.Tensor, qstats: torch.Tensor, T: int, block: int, scale: float,
                         top_p: float, n_sink: int = 1, n_local: int = 1, k_min: int = 0,
                         idx: torch.Tensor | None = None, count: torch.Tensor | None = None,
                         fmt: str = "int4", stream=None):
    """spa_select on quantised statistics (records in format fmt). Returns (idx, count)."""
    B, Hq, Lq, d = q.shape
    Hkv = qstats.shape[1]
    nb = -(-T // block)
    nq = -(-Lq // block)
    if idx is None:
        idx = torch.empty((B, Hq, nq, nb), device=q.device, dtype=torch.int32)
    if count is None:
        count = torch.empty((B, Hq, nq), device=q.device, dtype=torch.int32)
    _check("spa_select_quantized",
           lib().spa_select_quantized(_ptr(q), _dt(q), _ptr(qstats), _qfmt(fmt), B, Hq, Hkv, Lq,
                                      T, d, block, scale, top_p, n_sink, n_local, k_min, _ptr(idx),
                                      idx.shape[-1], _ptr(count), _stream(stream)))
    return idx, count


def spa_select_score_order(q: torch.Tensor, mean: torch.Tensor, var: torch.Tensor, block: int,
                           scale: float, top_p: float, n_sink: int = 1, n_local: int = 1,
                           k_min: int = 0, idx: torch.Tensor | None = None,
                           count: torch.Tensor | None = None, stream=None):
    """Prefill selection with the kept lists in traversal order. Returns (idx, count)."""
    B, Hq, L, d = q.shape
    Hkv = mean.shape[1]
    nb = -(-L // block)
    if idx is None:
        idx = torch.empty((B, Hq, nb, nb), device=q.device, dtype=torch.int32)
    if count is None:
        count = torch.empty((B, Hq, nb), device=q.device, dtype=torch.int32)
    _check("spa_select_score_order",
           lib().spa_select_score_order(_ptr(q), _dt(q), _ptr(mean), _ptr(var), B, Hq, Hkv, L, d,
                                        block, scale, top_p, n_sink, n_local, k_min, _ptr(idx),
                                        idx.shape[-1], _ptr(count), _stream(stream)))
    return idx, count


def spa_sparse_attn_prefill_early_stop(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                       block: int, idx: torch.Tensor, count: torch.Tensor,
                                       scale: float, tau: float, n_sink: int = 1, n_local: int = 1,
                                       out: torch.Tensor | None = None,
                                       lse: torch.Tensor | None = None, want_lse: bool = False,
                                       processed: torch.Tensor | None = None, stream=None):
    """Attention over the prefix of score-ordered lists kept by the early stop.
    Returns (out, lse or None, processed [B, Hq, nq] int32)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, L), device=q.device, dtype=torch.float32)
    if processed is None:
        processed = torch.empty(count.shape, device=q.device, dtype=torch.int32)
    _check("spa_sparse_attn_prefill_early_stop",
           lib().spa_sparse_attn_prefill_early_stop(_ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hq, Hkv,
                                                    L, d, block, _ptr(idx), idx.shape[-1],
                                                    _ptr(count), scale, n_sink, n_local, tau,
                                                    _ptr(out), _ptr(lse), _ptr(processed),
                                                    _stream(stream)))
    return out, lse, processed


def _hptr(t: torch.Tensor):
    if t.is_cuda:
        raise ValueError("spa_prefill_host takes host (CPU) tensors")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def spa_prefill_host_workspace_bytes(dtype: torch.dtype, B: int, Hq: int, Hkv: int, L: int,
                                     d: int, block: int) -> int:
    """Device workspace bytes spa_prefill_host needs for these sizes."""
    dt = SPA_BF16 if dtype == torch.bfloat16 else SPA_F32
    return int(lib().spa_prefill_host_workspace_bytes(dt, B, Hq, Hkv, L, d, block))


def spa_prefill_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int,
                     top_p: float, scale: float | None = None, n_sink: int = 1, n_local: int = 1,
                     k_min: int = 0, out: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The whole prefill path from host tensors (pinned for copy/compute overlap):
    q [B,Hq,L,d], k, v [B,Hkv,L,d] on the CPU -> out [B,Hq,L,d] on the CPU. Asynchronous
    on `stream`: synchronise it before reading out."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = torch.empty(q.shape, dtype=q.dtype, pin_memory=q.is_pinned())
    need = spa_prefill_host_workspace_bytes(q.dtype, B, Hq, Hkv, L, d, block)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    _check("spa_prefill_host",
           lib().spa_prefill_host(_hptr(q), _hptr(k), _hptr(v), _hptr(out), _dt(q), B, Hq, Hkv, L,
                                  d, block, scale, top_p, n_sink, n_local, k_min, _ptr(workspace),
                                  workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


def spa_pbs_workspace_bytes(B: int, Hq: int, Hkv: int, L: int, block: int) -> int:
    return int(lib().spa_pbs_workspace_bytes(B, Hq, Hkv, L, block))


def spa_pbs_permutation(q: torch.Tensor, k: torch.Tensor, block: int, seg_blocks: int,
                        scale: float, perm: torch.Tensor | None = None,
                        workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Segmented key permutation: perm [B, Hkv, L] int32 (original index per position)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if perm is None:
        perm = torch.empty((B, Hkv, L), device=q.device, dtype=torch.int32)
    need = spa_pbs_workspace_bytes(B, Hq, Hkv, L, block)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check("spa_pbs_permutation",
           lib().spa_pbs_permutation(_ptr(q), _ptr(k), _dt(q), B, Hq, Hkv, L, d, block, seg_blocks,
                                     scale, _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _ptr(perm),
                                     _stream(stream)))
    return perm


def spa_pbs_gather(x: torch.Tensor, perm: torch.Tensor, xp: torch.Tensor | None = None,
                   stream=None) -> torch.Tensor:
    """The permuted copy of K or V: xp[b, g, p] = x[b, g, perm[b, g, p]]."""
    B, Hkv, L, d = x.shape
    if xp is None:
        xp = torch.empty_like(x)
    _check("spa_pbs_gather",
           lib().spa_pbs_gather(_ptr(x), _dt(x), B, Hkv, L, d, _ptr(perm), _ptr(xp),
                                _stream(stream)))
    return xp


def spa_select_segperm(q: torch.Tensor, mean: torch.Tensor, var: torch.Tensor,
                       mean_p: torch.Tensor, var_p: torch.Tensor, block: int, seg_blocks: int,
                       scale: float, top_p: float, n_sink: int = 1, n_local: int = 1,
                       k_min: int = 0, idx: torch.Tensor | None = None,
                       count: torch.Tensor | None = None, stream=None):
    """Prefill selection on the segment-permuted layout. Returns (idx, count)."""
    B, Hq, L, d = q.shape
    Hkv = mean.shape[1]
    nb = -(-L // block)
    if idx is None:
        idx = torch.empty((B, Hq, nb, nb), device=q.device, dtype=torch.int32)
    if count is None:
        count = torch.empty((B, Hq, nb), device=q.device, dtype=torch.int32)
    _check("spa_select_segperm",
           lib().spa_select_segperm(_ptr(q), _dt(q), _ptr(mean), _ptr(var), _ptr(mean_p),
                                    _ptr(var_p), B, Hq, Hkv, L, d, block, seg_blocks, scale, top_p,
                                    n_sink, n_local, k_min, _ptr(idx), idx.shape[-1], _ptr(count),
                                    _stream(stream)))
    return idx, count


def spa_sparse_attn_prefill_segperm(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                    kp: torch.Tensor, vp: torch.Tensor, block: int, seg_blocks: int,
                                    idx: torch.Tensor, count: torch.Tensor, scale: float,
                                    out: torch.Tensor | None = None,
                                    lse: torch.Tensor | None = None, want_lse: bool = False,
                                    stream=None):
    """Block-sparse prefill on the segment-permuted layout. Returns (out, lse or None)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, L), device=q.device, dtype=torch.float32)
    _check("spa_sparse_attn_prefill_segperm",
           lib().spa_sparse_attn_prefill_segperm(_ptr(q), _ptr(k), _ptr(v), _ptr(kp), _ptr(vp),
                                                 _dt(q), B, Hq, Hkv, L, d, block, seg_blocks,
                                                 _ptr(idx), idx.shape[-1], _ptr(count), scale,
                                                 _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def spa_sparse_attn_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, block: int,
                            idx: torch.Tensor, count: torch.Tensor, scale: float,
                            out: torch.Tensor | None = None, lse: torch.Tensor | None = None,
                            want_lse: bool = False, stream=None):
    """Block-sparse causal attention over the kept blocks. Returns (out, lse or None)."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty((B, Hq, L), device=q.device, dtype=torch.float32)
    _check("spa_sparse_attn_prefill",
           lib().spa_sparse_attn_prefill(_ptr(q), _ptr(k), _ptr(v), _dt(q), B, Hq, Hkv, L, d,
                                         block, _ptr(idx), idx.shape[-1], _ptr(count), scale,
                                         _ptr(out), _ptr(lse), _stream(stream)))
    return out, lse


def spa_rla_block_states(k: torch.Tensor, v: torch.Tensor, block: int, blk_begin: int = 0,
                         blk_end: int | None = None, states: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Per-block linear-attention states W_j[e][c] = sum_u v_u[e] exp(k_u[c]):
    [B, Hkv, nb, d, d] bf16."""
    B, Hkv, T, d = k.shape
    nb = -(-T // block)
    if blk_end is None:
        blk_end = nb
    if states is None:
        states = torch.empty((B, Hkv, nb, d, d), device=k.device, dtype=torch.bfloat16)
    _check("spa_rla_block_states",
           lib().spa_rla_block_states(_ptr(k), _ptr(v), _dt(k), B, Hkv, T, d, block, blk_begin,
                                      blk_end, _ptr(states), _stream(stream)))
    return states


def spa_rla_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, states: torch.Tensor,
                    block: int, idx: torch.Tensor, count: torch.Tensor,
                    out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Residual Linear Attention branch of prefill: [B, Hq, L, d] fp32."""
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    if out is None:
        out = torch.empty((B, Hq, L, d), device=q.device, dtype=torch.float32)
    _check("spa_rla_prefill",
           lib().spa_rla_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(states), _dt(q), B, Hq, Hkv, L, d,
                                 block, _ptr(idx), idx.shape[-1], _ptr(count), _ptr(out),
                                 _stream(stream)))
    return out


def spa_rla_decode_state(kc: torch.Tensor, vc: torch.Tensor, tok_begin: int = 0,
                         tok_end: int | None = None, state: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """Adds sum_{t in [tok_begin, tok_end)} v_t exp(k_t)^T into state [B, Hkv, d, d]
    fp32 (a zeroed state is made when none is given)."""
    B, Hkv, T, d = kc.shape
    if tok_end is None:
        tok_end = T
    if state is None:
        state = torch.zeros((B, Hkv, d, d), device=kc.device, dtype=torch.float32)
    _check("spa_rla_decode_state",
           lib().spa_rla_decode_state(_ptr(kc), _ptr(vc), _dt(kc), B, Hkv, T, d, tok_begin,
                                      tok_end, _ptr(state), _stream(stream)))
    return state


def spa_rla_decode_workspace_bytes(B: int, Hq: int, Hkv: int, T: int, d: int, block: int) -> int:
    return int(lib().spa_rla_decode_workspace_bytes(B, Hq, Hkv, T, d, block))


def spa_sparse_attn_decode_rla(q: torch.Tensor, kc: torch.Tensor, vc: torch.Tensor,
                               state: torch.Tensor, block: int, idx: torch.Tensor,
                               count: torch.Tensor, scale: float,
                               workspace: torch.Tensor | None = None,
                               out: torch.Tensor | None = None,
                               out_rla: torch.Tensor | None = None, stream=None):
    """Decode attention plus the linear branch over the unkept blocks.
    Returns (out [B,Hq,1,d] bf16, out_rla [B,Hq,1,d] fp32)."""
    B, Hq, _, d = q.shape
    Hkv, T = kc.shape[1], kc.shape[2]
    if workspace is None:
        n = spa_rla_decode_workspace_bytes(B, Hq, Hkv, T, d, block)
        workspace = torch.empty((max(n, 16),), device=q.device, dtype=torch.uint8)
    if out is None:
        out = torch.empty_like(q)
    if out_rla is None:
        out_rla = torch.empty(q.shape, device=q.device, dtype=torch.float32)
    _check("spa_sparse_attn_decode_rla",
           lib().spa_sparse_attn_decode_rla(_ptr(q), _ptr(kc), _ptr(vc), _ptr(state), _dt(q), B,
                                            Hq, Hkv, T, d, block, _ptr(idx), idx.shape[-1],
                                            _ptr(count), scale, _ptr(workspace), _ptr(out),
                                            _ptr(out_rla), _stream(stream)))
    return out, out_rla


def spa_decode_workspace_bytes(B: int, Hq: int, Hkv: int, T: int, d: int, block: int) -> int:
    return int(lib().spa_decode_workspace_bytes(B, Hq, Hkv, T, d, block))


def spa_sparse_attn_decode(q: torch.Tensor, kc: torch.Tensor, vc: torch.Tensor, block: int,
                           idx: torch.Tensor, count: torch.Tensor, scale: float,
                           workspace: torch.Tensor | None = None,
                           out: torch.Tensor | None = None, stream=None):
    """Decode attention for one query per sequence: q [B,Hq,1,d] -> out [B,Hq,1,d]."""
    B, Hq, _, d = q.shape
    Hkv, T = kc.shape[1], kc.shape[2]
    if workspace is None:
        n = spa_decode_workspace_bytes(B, Hq, Hkv, T, d, block)
        workspace = torch.empty((max(n, 16),), device=q.device, dtype=torch.uint8)
    if out is None:
        out = torch.empty_like(q)
    _check("spa_sparse_attn_decode",
           lib().spa_sparse_attn_decode(_ptr(q), _ptr(kc), _ptr(vc), _dt(q), B, Hq, Hkv, T, d,
                                        block, _ptr(idx), idx.shape[-1], _ptr(count), scale,
                                        _ptr(workspace), _ptr(out), _stream(stream)))
    return out


def spa_selftest_wait_timeout(limit_us: int, stream=None) -> None:
    """Enqueues the bounded-wait self-test: a wait that nothing completes runs out
    after limit_us and records SPA_DEVERR_TIMEOUT (read it with spa_get_device_error)."""
    _check("spa_selftest_wait_timeout", lib().spa_selftest_wait_timeout(limit_us, _stream(stream)))


def spa_get_device_error() -> int:
    """Reads and clears the device error word (synchronises); 0 means no error."""
    code = ctypes.c_int(0)
    st = lib().spa_get_device_error(ctypes.byref(code))
    if st not in (0, 4):
        _check("spa_get_device_error", st)
    return code.value


def prefill(q, k, v, block: int, top_p: float, scale: float | None = None, n_sink: int = 1,
            n_local: int = 1, k_min: int = 0, want_lse: bool = False, stream=None):
    """The whole prefill path: block stats -> selection -> sparse attention.

    Returns dict(out, lse, idx, count, mean, var).
    """
    T = k.shape[2]
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    mean, var = spa_block_stats(k, block, stream=stream)
    idx, count = spa_select(q, mean, var, T, block, scale, top_p, n_sink, n_local, k_min,
                            stream=stream)
    out, lse = spa_sparse_attn_prefill(q, k, v, block, idx, count, scale, want_lse=want_lse,
                                       stream=stream)
    return {"out": out, "lse": lse, "idx": idx, "count": count, "mean": mean, "var": var}


def decode(q, kc, vc, block: int, top_p: float, mean=None, var=None, scale: float | None = None,
           n_sink: int = 1, n_local: int = 1, k_min: int = 0, workspace=None, stream=None):
    """One decode step: (stats, if not given) -> selection -> sparse decode attention."""
    T = kc.shape[2]
    scale = 1.0 / math.sqrt(q.shape[-1]) if scale is None else scale
    if mean is None or var is None:
        mean, var = spa_block_stats(kc, block, stream=stream)
    idx, count = spa_select(q, mean, var, T, block, scale, top_p, n_sink, n_local, k_min,
                            stream=stream)
    out = spa_sparse_attn_decode(q, kc, vc, block, idx, count, scale, workspace=workspace,
                                 stream=stream)
    return {"out": out, "idx": idx, "count": count, "mean": mean, "var": var}
