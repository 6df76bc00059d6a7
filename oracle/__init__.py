"""CPU oracle for selection-driven block-sparse causal attention (fp64).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline and reference (oracle-timing) legs of ``bench.py`` may import this
package. It shares no code with
the CUDA path and never imports it; the CUDA path never imports this.

The arithmetic lives in ``spa_oracle.c`` (plain C loops, fp64, OpenMP over
independent units); this module only compiles it with gcc and marshals numpy
arrays. Each function cites the passage it follows in its C counterpart.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_spa.so")
_lib = None
_lock = threading.Lock()

_P = ctypes.c_void_p
_I = ctypes.c_int
_D = ctypes.c_double
_I64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile ``spa_oracle.c`` into ``liboracle_spa.so`` (gcc, fp64, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall", "-Wextra", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    lib = ctypes.CDLL(path)
    lib.oracle_num_threads.restype = _I
    lib.oracle_block_stats.argtypes = [_P, _I, _I, _I, _I, _I, _I, _P, _P]
    lib.oracle_scores.argtypes = [_P, _I, _P, _P, _I, _I, _I, _I, _I, _I, _I, _D, _P]
    lib.oracle_select_from_scores.argtypes = [_P, _I, _I, _I, _I, _I, _D, _I, _I, _I,
                                              _P, _I, _P]
    lib.oracle_attention.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                                     _P, _I, _P, _D, _P, _I64, _P, _P]
    lib.oracle_rla.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I,
                               _P, _I, _P, _P, _I64, _P, _P]
    lib.oracle_rla_block_states.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _P]
    lib.oracle_early_stop.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _I, _P, _D, _I,
                                      _I, _D, _P, _P]
    lib.oracle_pbs_permutation.argtypes = [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _D, _P, _P]
    lib.oracle_attention_segperm.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P,
                                             _I, _P, _D, _P, _I64, _P, _P]
    lib.oracle_quantize_stats.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P]
    lib.oracle_dequantize_stats.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P]
    lib.oracle_quantize_stats_fp4.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P]
    lib.oracle_dequantize_stats_fp4.argtypes = [_P, _P, _P, _P, _I, _I, _I, _I, _P, _P]
    for f in ("oracle_block_stats", "oracle_scores", "oracle_select_from_scores",
              "oracle_attention", "oracle_rla", "oracle_rla_block_states",
              "oracle_quantize_stats", "oracle_dequantize_stats", "oracle_quantize_stats_fp4",
              "oracle_dequantize_stats_fp4", "oracle_early_stop",
              "oracle_pbs_permutation", "oracle_attention_segperm"):
        getattr(lib, f).restype = _I
    return lib


def use_library(path: str | None):
    """Point this module at another build of the oracle (``None``: the default).

    Used by the mutation tests, which compile deliberately broken copies of the
    oracle source to show that the pins catch them.
    """
    global _lib
    with _lock:
        _lib = _bind(path) if path else None


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def num_threads() -> int:
    """Threads the oracle's parallel loops use (OpenMP's default team size)."""
    return int(_load().oracle_num_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _inp(x: np.ndarray, dtype: str) -> tuple[np.ndarray, int]:
    if dtype == "bf16":
        return np.ascontiguousarray(x, dtype=np.uint16), 1
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32), 0
    raise ValueError(dtype)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def block_stats(k: np.ndarray, dtype: str, block: int):
    """Per-block key mean and population variance (fp64). k: [B,Hkv,T,d]."""
    k, isb = _inp(k, dtype)
    B, Hkv, T, d = k.shape
    nb = -(-T // block)
    mean = np.empty((B, Hkv, nb, d), np.float64)
    var = np.empty_like(mean)
    _check(_load().oracle_block_stats(_ptr(k), isb, B, Hkv, T, d, block, _ptr(mean), _ptr(var)),
           "block_stats")
    return mean, var


def scores(q: np.ndarray, dtype: str, mean: np.ndarray, var: np.ndarray, T: int, block: int,
           scale: float) -> np.ndarray:
    """Log Taylor block scores [B,Hq,nq,nb] (fp64); -inf beyond the causal limit."""
    q, isb = _inp(q, dtype)
    B, Hq, Lq, d = q.shape
    Hkv = mean.shape[1]
    nb = -(-T // block)
    nq = -(-Lq // block)
    mean = np.ascontiguousarray(mean, np.float64)
    var = np.ascontiguousarray(var, np.float64)
    l = np.empty((B, Hq, nq, nb), np.float64)
    _check(_load().oracle_scores(_ptr(q), isb, _ptr(mean), _ptr(var), B, Hq, Hkv, Lq, T, d,
                                 block, float(scale), _ptr(l)), "scores")
    return l


def select_from_scores(l: np.ndarray, Lq: int, T: int, block: int, top_p: float, n_sink: int = 1,
                       n_local: int = 1, k_min: int = 0, cap: int | None = None):
    """Dual top-p cut over given log scores. Returns (idx [B,Hq,nq,cap] int32, count int32)."""
    l = np.ascontiguousarray(l, np.float64)
    B, Hq, nq, nb = l.shape
    cap = nb if cap is None else cap
    idx = np.empty((B, Hq, nq, cap), np.int32)
    count = np.empty((B, Hq, nq), np.int32)
    _check(_load().oracle_select_from_scores(_ptr(l), B, Hq, Lq, T, block, float(top_p), n_sink,
                                             n_local, k_min, _ptr(idx), cap, _ptr(count)),
           "select")
    return idx, count


def select(q, k, dtype: str, block: int, scale: float, top_p: float, n_sink: int = 1,
           n_local: int = 1, k_min: int = 0, cap: int | None = None):
    """Stats -> pooled scores -> cut. Returns dict(mean, var, scores, idx, count)."""
    mean, var = block_stats(k, dtype, block)
    T = k.shape[2]
    l = scores(q, dtype, mean, var, T, block, scale)
    idx, count = select_from_scores(l, q.shape[2], T, block, top_p, n_sink, n_local, k_min, cap)
    return {"mean": mean, "var": var, "scores": l, "idx": idx, "count": count}


def attention(q, k, v, dtype: str, block: int, idx: np.ndarray, count: np.ndarray, scale: float,
              rows: np.ndarray | None = None):
    """Masked dense softmax attention (fp64), all rows or the flat row ids ``rows``.

    Returns (out, lse): out [B,Hq,Lq,d] (or [len(rows), d]), lse likewise without d.
    """
    q, isb = _inp(q, dtype)
    k, _ = _inp(k, dtype)
    v, _ = _inp(v, dtype)
    B, Hq, Lq, d = q.shape
    Hkv, T = k.shape[1], k.shape[2]
    idx = np.ascontiguousarray(idx, np.int32)
    count = np.ascontiguousarray(count, np.int32)
    cap = idx.shape[-1]
    if rows is None:
        n = B * Hq * Lq
        out = np.empty((B, Hq, Lq, d), np.float64)
        lse = np.empty((B, Hq, Lq), np.float64)
        rp = None
    else:
        rows = np.ascontiguousarray(rows, np.int64)
        n = rows.size
        out = np.empty((n, d), np.float64)
        lse = np.empty((n,), np.float64)
        rp = _ptr(rows)
    _check(_load().oracle_attention(_ptr(q), _ptr(k), _ptr(v), isb, B, Hq, Hkv, Lq, T, d, block,
                                    _ptr(idx), cap, _ptr(count), float(scale), rp, n, _ptr(out),
                                    _ptr(lse)), "attention")
    return out, lse


def rla(q, k, v, dtype: str, block: int, idx: np.ndarray, count: np.ndarray,
        rows: np.ndarray | None = None):
    """Residual Linear Attention (fp64): for each query row, the linear attention
    with phi = exp over the causal tokens of the blocks its kept list leaves out.

    Returns (out, mag): out [B,Hq,Lq,d] (or [len(rows), d]); mag is the same sum
    with |v| in place of v (the magnitude that rounding errors scale with).
    """
    q, isb = _inp(q, dtype)
    k, _ = _inp(k, dtype)
    v, _ = _inp(v, dtype)
    B, Hq, Lq, d = q.shape
    Hkv, T = k.shape[1], k.shape[2]
    idx = np.ascontiguousarray(idx, np.int32)
    count = np.ascontiguousarray(count, np.int32)
    cap = idx.shape[-1]
    if rows is None:
        n = B * Hq * Lq
        out = np.empty((B, Hq, Lq, d), np.float64)
        rp = None
    else:
        rows = np.ascontiguousarray(rows, np.int64)
        n = rows.size
        out = np.empty((n, d), np.float64)
        rp = _ptr(rows)
    mag = np.empty_like(out)
    _check(_load().oracle_rla(_ptr(q), _ptr(k), _ptr(v), isb, B, Hq, Hkv, Lq, T, d, block,
                              _ptr(idx), cap, _ptr(count), rp, n, _ptr(out), _ptr(mag)), "rla")
    return out, mag


def rla_block_states(k, v, dtype: str, block: int) -> np.ndarray:
    """Per-block states W_j[e][c] = sum_{u in block j} v_u,e exp(k_u,c), fp64
    [B, Hkv, nb, d, d]."""
    k, isb = _inp(k, dtype)
    v, _ = _inp(v, dtype)
    B, Hkv, T, d = k.shape
    nb = -(-T // block)
    out = np.empty((B, Hkv, nb, d, d), np.float64)
    _check(_load().oracle_rla_block_states(_ptr(k), _ptr(v), isb, B, Hkv, T, d, block, _ptr(out)),
           "rla_block_states")
    return out


def quantize_stats(mean: np.ndarray, var: np.ndarray, fmt: str = "int4") -> dict:
    """Microscale block statistics (SpotAttention, section 4): INT4 (fmt "int4", the
    format documented at oracle_quantize_stats) or FP4 E2M1 (fmt "fp4", documented at
    oracle_quantize_stats_fp4). Returns codes cm, cv shaped like mean (INT4: int8 and
    uint8 values; FP4: uint8 4-bit patterns), per-32-feature exponents km, kv (int8)
    [B, Hkv, nb, d / 32], and the format."""
    mean = np.ascontiguousarray(mean, np.float64)
    var = np.ascontiguousarray(var, np.float64)
    B, Hkv, nb, d = mean.shape
    km = np.empty((B, Hkv, nb, d // 32), np.int8)
    kv = np.empty_like(km)
    cv = np.empty(mean.shape, np.uint8)
    if fmt == "int4":
        cm = np.empty(mean.shape, np.int8)
        fn = _load().oracle_quantize_stats
    elif fmt == "fp4":
        cm = np.empty(mean.shape, np.uint8)
        fn = _load().oracle_quantize_stats_fp4
    else:
        raise ValueError(f"unknown format {fmt!r}")
    _check(fn(_ptr(mean), _ptr(var), B, Hkv, nb, d, _ptr(cm), _ptr(cv), _ptr(km), _ptr(kv)),
           "quantize_stats")
    return {"cm": cm, "cv": cv, "km": km, "kv": kv, "fmt": fmt}


def dequantize_stats(qs: dict):
    """(mean, var) fp64 from quantize_stats' codes: code * 2^k (INT4) or
    E2M1(code) * 2^k (FP4)."""
    fmt = qs.get("fmt", "int4")
    cm = np.ascontiguousarray(qs["cm"], np.int8 if fmt == "int4" else np.uint8)
    cv = np.ascontiguousarray(qs["cv"], np.uint8)
    km = np.ascontiguousarray(qs["km"], np.int8)
    kv = np.ascontiguousarray(qs["kv"], np.int8)
    B, Hkv, nb, d = cm.shape
    mean = np.empty(cm.shape, np.float64)
    var = np.empty(cm.shape, np.float64)
    fn = _load().oracle_dequantize_stats if fmt == "int4" else _load().oracle_dequantize_stats_fp4
    _check(fn(_ptr(cm), _ptr(cv), _ptr(km), _ptr(kv), B, Hkv, nb, d, _ptr(mean), _ptr(var)),
           "dequantize_stats")
    return mean, var


def select_quantized(q, k, dtype: str, block: int, scale: float, top_p: float, n_sink: int = 1,
                     n_local: int = 1, k_min: int = 0, fmt: str = "int4"):
    """The selection of `select` on quantised statistics: stats -> quantize (fmt) ->
    dequantize -> scores -> cut."""
    mean, var = block_stats(k, dtype, block)
    qs = quantize_stats(mean, var, fmt)
    dm, dv = dequantize_stats(qs)
    Lq, T = q.shape[2], k.shape[2]
    l = scores(q, dtype, dm, dv, T, block, scale)
    idx, count = select_from_scores(l, Lq, T, block, top_p, n_sink, n_local, k_min)
    return {"mean": mean, "var": var, "q": qs, "scores": l, "idx": idx, "count": count}


def score_order(sel: dict, Lq: int, T: int, block: int, n_sink: int = 1, n_local: int = 1):
    """The kept lists of `select` in traversal order (S2O, section 2): the local
    blocks (the own block first, descending), the sink blocks (ascending), then the
    kept residual blocks by descending fp32 score, equal scores by ascending index.
    Returns (idx, count) with the same counts."""
    idx, count, l = sel["idx"], sel["count"], sel["scores"]
    out = np.full_like(idx, -1)
    B, Hq, nq, cap = idx.shape
    for b in range(B):
        for h in range(Hq):
            for i in range(nq):
                c = int(count[b, h, i])
                lst = [int(j) for j in idx[b, h, i, :c]]
                last_row = min((i + 1) * block, Lq)
                jmax = (T - Lq + last_row - 1) // block
                # reserved ranges as the cut defines them: sink [0, r_lo), local
                # [r_hi, jmax]; where they would overlap the sink takes precedence
                r_lo = min(n_sink, jmax + 1)
                r_hi = max(r_lo, jmax - n_local + 1)
                local = sorted([j for j in lst if j >= r_hi], reverse=True)
                sink = sorted([j for j in lst if j < r_lo])
                res = [j for j in lst if r_lo <= j < r_hi]
                res.sort(key=lambda j: (-float(np.float32(l[b, h, i, j])), j))
                order = local + sink + res
                out[b, h, i, :c] = order
    return out, count.copy()


def early_stop(q, k, dtype: str, block: int, idx: np.ndarray, count: np.ndarray, scale: float,
               tau: float, n_sink: int = 1, n_local: int = 1):
    """S2O's monotone-gain early stop over score-ordered lists (prefill). Returns
    (processed [B,Hq,nq] int32, ratios [B,Hq,nq,cap] fp64: R_n per position, -1 past
    the stop)."""
    q, isb = _inp(q, dtype)
    k, _ = _inp(k, dtype)
    B, Hq, Lq, d = q.shape
    Hkv, T = k.shape[1], k.shape[2]
    idx = np.ascontiguousarray(idx, np.int32)
    count = np.ascontiguousarray(count, np.int32)
    cap = idx.shape[-1]
    processed = np.empty(count.shape, np.int32)
    ratios = np.empty(idx.shape, np.float64)
    _check(_load().oracle_early_stop(_ptr(q), _ptr(k), isb, B, Hq, Hkv, Lq, T, d, block, _ptr(idx),
                                     cap, _ptr(count), float(scale), n_sink, n_local, float(tau),
                                     _ptr(processed), _ptr(ratios)), "early_stop")
    return processed, ratios


def pbs_permutation(q, k, dtype: str, block: int, seg_blocks: int, scale: float,
                    return_importance: bool = False):
    """Segmented key permutation (PBS, sections 2-3; reading in spa_oracle.c): keys
    sorted inside each segment by the mean-pooled causal softmax weights of the last
    query block's rows (all query heads of the kv-group).
    Returns perm [B, Hkv, L] int32, the original index of the key at each permuted
    position, and with ``return_importance`` also the fp64 importance [B, Hkv, L]."""
    q, isb = _inp(q, dtype)
    k, _ = _inp(k, dtype)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    perm = np.empty((B, Hkv, L), np.int32)
    imp = np.empty((B, Hkv, L), np.float64)
    _check(_load().oracle_pbs_permutation(_ptr(q), _ptr(k), isb, B, Hq, Hkv, L, d, block, seg_blocks,
                                          float(scale), _ptr(perm), _ptr(imp)), "pbs_permutation")
    return (perm, imp) if return_importance else perm


def permute(x: np.ndarray, perm: np.ndarray) -> np.ndarray:
    """x [B, Hkv, L, d] in the permuted layout: row p of (b, g) is x[b, g, perm[b, g, p]]."""
    return np.take_along_axis(x, perm[..., None].astype(np.int64), axis=2)


def select_segperm(q, k, dtype: str, block: int, seg_blocks: int, scale: float, top_p: float,
                   n_sink: int = 1, n_local: int = 1, k_min: int = 0, perm=None):
    """The selection on the segment-permuted layout: a query block scores the blocks
    of earlier segments on the permuted keys' statistics and the blocks of its own
    segment on the original ones; then the same cut."""
    if perm is None:
        perm = pbs_permutation(q, k, dtype, block, seg_blocks, scale)
    kp = permute(np.asarray(k), perm)
    mean, var = block_stats(k, dtype, block)
    mp, vp = block_stats(kp, dtype, block)
    L = q.shape[2]
    lo = scores(q, dtype, mean, var, L, block, scale)
    lp = scores(q, dtype, mp, vp, L, block, scale)
    nq = lo.shape[2]
    seg0 = (np.arange(nq) // seg_blocks) * seg_blocks          # first block of the own segment
    use_p = np.arange(lo.shape[3])[None, :] < seg0[:, None]      # [nq, nb]
    l = np.where(use_p[None, None], lp, lo)
    idx, count = select_from_scores(l, L, L, block, top_p, n_sink, n_local, k_min)
    return {"perm": perm, "mean": mean, "var": var, "mean_p": mp, "var_p": vp, "scores": l,
            "idx": idx, "count": count}


def attention_segperm(q, k, v, dtype: str, block: int, seg_blocks: int, perm: np.ndarray,
                      idx: np.ndarray, count: np.ndarray, scale: float,
                      rows: np.ndarray | None = None):
    """Masked softmax attention for lists on the segment-permuted layout (fp64);
    returns (out, lse) like `attention`."""
    q, isb = _inp(q, dtype)
    k, _ = _inp(k, dtype)
    v, _ = _inp(v, dtype)
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    perm = np.ascontiguousarray(perm, np.int32)
    idx = np.ascontiguousarray(idx, np.int32)
    count = np.ascontiguousarray(count, np.int32)
    cap = idx.shape[-1]
    if rows is None:
        n = B * Hq * L
        out = np.empty((B, Hq, L, d), np.float64)
        lse = np.empty((B, Hq, L), np.float64)
        rp = None
    else:
        rows = np.ascontiguousarray(rows, np.int64)
        n = rows.size
        out = np.empty((n, d), np.float64)
        lse = np.empty((n,), np.float64)
        rp = _ptr(rows)
    _check(_load().oracle_attention_segperm(_ptr(q), _ptr(k), _ptr(v), isb, B, Hq, Hkv, L, d, block,
                                            seg_blocks, _ptr(perm), _ptr(idx), cap, _ptr(count),
                                            float(scale), rp, n, _ptr(out), _ptr(lse)),
           "attention_segperm")
    return out, lse


def full_lists(B: int, Hq: int, Lq: int, T: int, block: int):
    """Kept lists that keep every causal block (dense causal attention)."""
    nb = -(-T // block)
    nq = -(-Lq // block)
    idx = np.full((B, Hq, nq, nb), -1, np.int32)
    count = np.empty((B, Hq, nq), np.int32)
    for i in range(nq):
        last_row = min((i + 1) * block, Lq)
        jmax = (T - Lq + last_row - 1) // block
        idx[:, :, i, :jmax + 1] = np.arange(jmax + 1, dtype=np.int32)
        count[:, :, i] = jmax + 1
    return idx, count
