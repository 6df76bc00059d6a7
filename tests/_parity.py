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
