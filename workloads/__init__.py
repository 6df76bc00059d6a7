"""Seeded synthetic workloads for selection-driven block-sparse attention.

This module only draws inputs. It holds none of the method's arithmetic (no
statistics, scores, selection or attention), so both sides of every parity check
can take their inputs from it: the CPU oracle (through the tests) and the CUDA
path (through the binding and ``bench.py``).

Recipe (the same for every workload; the sizes and knobs differ):

* Values are fp32 draws from N(0, 1) (numpy ``PCG64``), one independent stream per
  (tensor, batch, head), so any (b, head) slice can be drawn on its own and the
  draws can run on several threads.
* Heavy hitters: per (b, kv-head) a fraction ``hh_frac`` of key positions is
  chosen uniformly without replacement and set to ``4*sqrt(d)*u + eps``, where u
  is a random unit direction shared by the kv-head and eps is the position's own
  N(0, I) draw. The planted part has four times the norm of a typical key.
* Local-window bias (``local_window > 0``): every key j is nudged by
  ``0.5*sqrt(d)*unit(W_j)``, where ``W_j`` sums the queries of its kv-group at
  positions j .. j+local_window-1, so a key leans toward the queries that see it
  from close by.
* bf16 workloads round the fp32 draws to bf16 (round to nearest, ties to even);
  both sides then read the same bf16 values.
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = ["Workload", "WORKLOADS", "PARITY_WORKLOADS", "generate", "widen",
           "bf16_bits", "bf16_round", "n_threads"]

_Q, _K, _V, _HH = 1, 2, 3, 4


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic problem: shapes, block size, selection knobs and data recipe."""
    name: str
    mode: str            # "prefill" (Lq == T) or "decode" (Lq == 1, query at position T-1)
    dtype: str           # "f32" or "bf16": storage and input type of Q, K, V
    B: int
    Hq: int
    Hkv: int
    T: int               # key/value length (prefill: also the query length)
    d: int
    block: int
    top_p: float
    n_sink: int = 1
    n_local: int = 1
    k_min: int = 0
    hh_frac: float = 0.0
    local_window: int = 0
    seed: int = 0

    @property
    def Lq(self) -> int:
        return self.T if self.mode == "prefill" else 1

    @property
    def nb(self) -> int:
        return -(-self.T // self.block)

    @property
    def nq(self) -> int:
        return -(-self.Lq // self.block) if self.mode == "prefill" else 1

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def scale(self) -> float:
        """Softmax scale 1/sqrt(d), rounded to fp32 (both sides use this value)."""
        return float(np.float32(1.0 / math.sqrt(self.d)))

    def shapes(self):
        return {"q": (self.B, self.Hq, self.Lq, self.d),
                "k": (self.B, self.Hkv, self.T, self.d),
                "v": (self.B, self.Hkv, self.T, self.d)}

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def _w(cid, name, **kw):
    return Workload(name=name, seed=20261202 + cid, **kw)


#: The five headline workloads, keyed by number (1 = tiny fp32, 5 = decode).
WORKLOADS = {
    1: _w(1, "prefill_f32_L1024_H1_d64_blk64", mode="prefill", dtype="f32", B=1, Hq=1,
          Hkv=1, T=1024, d=64, block=64, top_p=0.9),
    2: _w(2, "prefill_bf16_L8192_H32x8_d128_blk64", mode="prefill", dtype="bf16", B=1,
          Hq=32, Hkv=8, T=8192, d=128, block=64, top_p=0.95, hh_frac=0.01),
    3: _w(3, "prefill_bf16_L32768_H32x8_d128_blk128", mode="prefill", dtype="bf16", B=1,
          Hq=32, Hkv=8, T=32768, d=128, block=128, top_p=0.9, hh_frac=0.005,
          local_window=512),
    4: _w(4, "prefill_bf16_L131072_H32x8_d128_blk128", mode="prefill", dtype="bf16", B=1,
          Hq=32, Hkv=8, T=131072, d=128, block=128, top_p=0.9, hh_frac=0.002),
    5: _w(5, "decode_bf16_B16_T131072_H32x8_d128_blk16", mode="decode", dtype="bf16", B=16,
          Hq=32, Hkv=8, T=131072, d=128, block=16, top_p=0.9, hh_frac=0.002),
}

#: Small versions of the same recipes that the oracle finishes in seconds; they
#: span several tiles and end on a ragged (partial) block.
PARITY_WORKLOADS = {
    "p_bf16_blk128": _w(103, "prefill_bf16_L1000_H8x2_d128_blk128", mode="prefill",
                        dtype="bf16", B=2, Hq=8, Hkv=2, T=1000, d=128, block=128,
                        top_p=0.9, hh_frac=0.005, local_window=256),
    "p_bf16_blk64": _w(102, "prefill_bf16_L1000_H8x2_d128_blk64", mode="prefill",
                       dtype="bf16", B=1, Hq=8, Hkv=2, T=1000, d=128, block=64,
                       top_p=0.95, hh_frac=0.01),
    "p_f32_d64": _w(101, "prefill_f32_L1000_H2x1_d64_blk64", mode="prefill", dtype="f32",
                    B=1, Hq=2, Hkv=1, T=1000, d=64, block=64, top_p=0.9),
    "p_f32_d128": _w(104, "prefill_f32_L700_H4x2_d128_blk128", mode="prefill", dtype="f32",
                     B=1, Hq=4, Hkv=2, T=700, d=128, block=128, top_p=0.9, hh_frac=0.01),
    "d_bf16_blk16": _w(105, "decode_bf16_B3_T1000_H8x2_d128_blk16", mode="decode",
                       dtype="bf16", B=3, Hq=8, Hkv=2, T=1000, d=128, block=16,
                       top_p=0.9, hh_frac=0.01),
    "d_bf16_blk64": _w(106, "decode_bf16_B2_T3000_H8x2_d128_blk64", mode="decode",
                       dtype="bf16", B=2, Hq=8, Hkv=2, T=3000, d=128, block=64,
                       top_p=0.9, hh_frac=0.01),
}


def n_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Storage form -> fp32 values (exact: bf16 widens to fp32 without rounding)."""
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32)
    return (np.asarray(x, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 values rounded to the nearest bf16 value, returned as fp32."""
    return widen(bf16_bits(x), "bf16")


def _rng(w: Workload, tensor: int, b: int, h: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([w.seed, tensor, b, h])))


def _q_slice(w: Workload, b: int, h: int) -> np.ndarray:
    """Query rows of (b, h) as fp32 values after storage rounding."""
    x = _rng(w, _Q, b, h).standard_normal((w.Lq, w.d), dtype=np.float32)
    return bf16_round(x) if w.dtype == "bf16" else x


def _kv_slice(w: Workload, b: int, g: int, qgroup: np.ndarray | None):
    d = w.d
    k = _rng(w, _K, b, g).standard_normal((w.T, d), dtype=np.float32)
    v = _rng(w, _V, b, g).standard_normal((w.T, d), dtype=np.float32)
    if w.hh_frac > 0:
        r = _rng(w, _HH, b, g)
        n_hh = min(w.T, int(math.ceil(w.hh_frac * w.T)))
        pos = r.choice(w.T, size=n_hh, replace=False)
        u = r.standard_normal(d)
        u /= np.linalg.norm(u)
        k[pos] += np.float32(4.0 * math.sqrt(d)) * u.astype(np.float32)
    if w.local_window > 0 and qgroup is not None:
        # W_j = sum_{t=j}^{min(j+win-1, T-1)} sum_{h in group} q_{h,t}
        qs = qgroup.astype(np.float64).sum(axis=0)                    # [T, d]
        c = np.concatenate([np.zeros((1, d)), np.cumsum(qs, axis=0)])  # [T+1, d]
        j = np.arange(w.T)
        hi = np.minimum(j + w.local_window, w.T)
        W = c[hi] - c[j]
        nrm = np.linalg.norm(W, axis=1, keepdims=True)
        nrm[nrm == 0] = 1.0
        k += (0.5 * math.sqrt(d) * W / nrm).astype(np.float32)
    return k, v


def generate(w: Workload, heads: list[tuple[int, int]] | None = None, threads: int | None = None):
    """Draw Q, K, V for ``w`` in storage form.

    Returns ``{"q", "k", "v"}``: float32 arrays for ``f32`` workloads, uint16 bf16
    bit patterns for ``bf16`` workloads, in the layouts ``[B,Hq,Lq,d]`` and
    ``[B,Hkv,T,d]``.

    ``heads`` restricts the draw to a list of (b, kv-head) units (the other
    slices are left zero); every drawn slice is identical to the full draw.
    """
    sh = w.shapes()
    sdt = np.float32 if w.dtype == "f32" else np.uint16
    out = {n: np.zeros(s, dtype=sdt) for n, s in sh.items()}
    units = heads if heads is not None else [(b, g) for b in range(w.B) for g in range(w.Hkv)]
    G = w.G

    def store(name, idx, x):
        out[name][idx] = x if w.dtype == "f32" else bf16_bits(x)

    def one(unit):
        b, g = unit
        qg = [_q_slice(w, b, h) for h in range(g * G, (g + 1) * G)]
        for j, h in enumerate(range(g * G, (g + 1) * G)):
            store("q", (b, h), qg[j])
        k, v = _kv_slice(w, b, g, np.stack(qg) if w.local_window > 0 else None)
        store("k", (b, g), k)
        store("v", (b, g), v)

    nt = threads or n_threads()
    if nt > 1 and len(units) > 1:
        with ThreadPoolExecutor(min(nt, len(units))) as ex:
            list(ex.map(one, units))
    else:
        for u in units:
            one(u)
    return out
