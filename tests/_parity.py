"""Helpers shared by the GPU parity tests: device upload of the seeded inputs and
the kept-list comparison with near-tie accounting.

Comparison rule for kept lists: a (b, h, query-block) list must equal the
oracle's exactly, unless the difference is an excused near tie:
  (i)  every block in the symmetric difference has a score within 1e-5 relative
       of the oracle's last kept residual score, or
  (ii) the oracle's cumulative mass before or after its crossing block lies
       within 1e-5 relative of top_p.
Excused cases are counted and reported; anything else fails.
"""
from __future__ import annotations

import numpy as np
import torch

REL = 1e-5


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def to_host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()


def _jmax(i, Lq, T, block):
    last_row = min((i + 1) * block, Lq)
    return (T - Lq + last_row - 1) // block


def compare_lists(g_idx, g_cnt, o_idx, o_cnt, o_scores, top_p, n_sink, n_local, Lq, T, block):
    """Returns dict(units, equal, excused, unexcused=[(b,h,i,gpu,oracle)])."""
    B, Hq, nq = o_cnt.shape
    res = {"units": B * Hq * nq, "equal": 0, "excused": 0, "unexcused": []}
    same_cnt = g_cnt == o_cnt
    for b in range(B):
        for h in range(Hq):
            for i in range(nq):
                gc, oc = int(g_cnt[b, h, i]), int(o_cnt[b, h, i])
                if same_cnt[b, h, i] and np.array_equal(g_idx[b, h, i, :gc], o_idx[b, h, i, :oc]):
                    res["equal"] += 1
                    continue
                gs, os_ = set(g_idx[b, h, i, :gc].tolist()), set(o_idx[b, h, i, :oc].tolist())
                if _excused(gs, os_, o_scores[b, h, i], top_p, n_sink, n_local, i, Lq, T, block):
                    res["excused"] += 1
                else:
                    res["unexcused"].append((b, h, i, sorted(gs), sorted(os_)))
    return res


def _excused(gs, os_, scores, top_p, n_sink, n_local, i, Lq, T, block):
    jmax = _jmax(i, Lq, T, block)
    resid = [j for j in range(jmax + 1) if not (j < n_sink or j > jmax - n_local)]
    kept = [j for j in resid if j in os_]
    sym = gs ^ os_
    if not resid or not kept or any(j not in resid for j in sym):
        return False
    s32 = {j: np.float32(scores[j]) for j in resid}
    order = sorted(resid, key=lambda j: (-s32[j], j))
    l_cut = float(s32[order[len(kept) - 1]])
    if all(abs(float(s32[j]) - l_cut) <= REL * max(1.0, abs(l_cut)) for j in sym):
        return True
    w = np.array([float(s32[j]) for j in order], np.float64)
    w = np.exp(w - w.max())
    w /= w.sum()
    before = np.concatenate([[0.0], np.cumsum(w)])
    nk = len(kept)
    near = [before[nk - 1], before[nk]] if nk <= len(order) else [before[nk - 1]]
    return any(abs(c / top_p - 1.0) <= REL for c in near)


def sample_rows(B, Hq, L, block, n, seed):
    """Flat row ids (b*Hq + h)*L + t: block edges, the first and last rows, and uniform rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    for bh in rng.choice(B * Hq, size=min(B * Hq, max(2, n // 8)), replace=False):
        for t in (0, min(L - 1, block - 1), min(L - 1, block), L - 1, max(0, L - block)):
            rows.add(int(bh) * L + t)
    while len(rows) < n:
        rows.add(int(rng.integers(0, B * Hq)) * L + int(rng.integers(0, L)))
    return np.array(sorted(rows), np.int64)


# ------------------------------------------------------------------ quantised statistics records
# Record layout of spa_quantize_block_stats (include/spa.h): d/2 bytes of mean codes
# (two per byte, even feature in the low nibble, signed), d/2 bytes of variance
# codes (unsigned), d/32 int8 mean exponents, d/32 int8 variance exponents.

def pack_qstats(qs: dict) -> np.ndarray:
    cm = qs["cm"].astype(np.int16) & 15
    cv = qs["cv"].astype(np.int16) & 15
    B, Hkv, nb, d = cm.shape
    rec = np.empty((B, Hkv, nb, d + d // 16), np.uint8)
    rec[..., :d // 2] = (cm[..., 0::2] | (cm[..., 1::2] << 4)).astype(np.uint8)
    rec[..., d // 2:d] = (cv[..., 0::2] | (cv[..., 1::2] << 4)).astype(np.uint8)
    rec[..., d:d + d // 32] = qs["km"].view(np.uint8)
    rec[..., d + d // 32:] = qs["kv"].view(np.uint8)
    return rec


def unpack_qstats(rec: np.ndarray, d: int, fmt: str = "int4") -> dict:
    rec = np.asarray(rec, np.uint8)
    lo_m, hi_m = rec[..., :d // 2] & 15, rec[..., :d // 2] >> 4
    lo_v, hi_v = rec[..., d // 2:d] & 15, rec[..., d // 2:d] >> 4
    cm = np.empty(rec.shape[:-1] + (d,), np.int16)
    cm[..., 0::2], cm[..., 1::2] = lo_m, hi_m
    # INT4 mean codes are two's-complement nibbles; FP4 codes stay 4-bit patterns
    cm = np.where(cm >= 8, cm - 16, cm).astype(np.int8) if fmt == "int4" else cm.astype(np.uint8)
    cv = np.empty(rec.shape[:-1] + (d,), np.uint8)
    cv[..., 0::2], cv[..., 1::2] = lo_v, hi_v
    return {"cm": cm, "cv": cv, "km": rec[..., d:d + d // 32].view(np.int8),
            "kv": rec[..., d + d // 32:].view(np.int8)}


E2M1_MIDPOINTS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def quant_ambiguous(mean: np.ndarray, var: np.ndarray, qs: dict, rel: float = 1e-5) -> np.ndarray:
    """Per 32-feature group: True where the oracle's quantisation decision is a near
    tie for fp32 statistics that differ in rounding order: a value within `rel` of a
    rounding boundary (INT4: a half step; FP4: a midpoint of the E2M1 grid, or zero,
    where the sign bit decides), or the group maximum within `rel` of a scale
    boundary. [B, Hkv, nb, d / 32], for mean or variance."""
    fmt = qs.get("fmt", "int4")
    tops = (7.0, 15.0) if fmt == "int4" else (6.0, 6.0)
    out = []
    for x, k, top in ((np.abs(mean.astype(np.float32).astype(np.float64)), qs["km"], tops[0]),
                      (var.astype(np.float32).astype(np.float64), qs["kv"], tops[1])):
        B, Hkv, nb, d = x.shape
        step = np.ldexp(1.0, k.astype(np.int64)).repeat(32, axis=-1)
        t = x / step
        tol = rel * np.maximum(1.0, t)
        if fmt == "int4":
            near = np.abs(t - np.floor(t) - 0.5) <= tol
        else:
            near = (np.abs(t[..., None] - E2M1_MIDPOINTS).min(-1) <= tol) | (t <= rel)
        near_code = near.reshape(B, Hkv, nb, d // 32, 32).any(-1)
        amax = x.reshape(B, Hkv, nb, d // 32, 32).max(-1)
        kk = k.astype(np.int64)
        near_scale = ((np.abs(amax / (top * np.ldexp(1.0, kk)) - 1) <= rel) |
                      (np.abs(amax / (top * np.ldexp(1.0, kk - 1)) - 1) <= rel))
        out.append(near_code | near_scale)
    return out[0] | out[1]
