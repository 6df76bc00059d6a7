"""Parity of the score-ordered traversal with S2O's monotone-gain early stop
("S2O - Vroege Stoppering voor Sparse Attention via Online Permutatie", sections
2-3) with the CPU oracle.

The stop is an integer decided by floating point: the kernel decides on its fp32
online-softmax state, the oracle in fp64. Processed counts must be equal unless the
oracle's ratio at the first position where the two differ lies within 1e-4
(relative) of tau. Outputs are compared with the oracle's attention over the
GPU's processed prefix of each list (max-abs 2e-2, the bf16 tolerance).
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_stats_b200 as spa
from tests._parity import compare_lists, to_dev, to_host
from workloads import PARITY_WORKLOADS, generate

pytestmark = pytest.mark.gpu

TOL = 2e-2
REL_TAU = 1e-4

_cache = {}


def inputs(w):
    key = (w.name, w.T, w.B, w.block, w.Hq, w.Hkv)
    if key not in _cache:
        x = generate(w)
        _cache.clear()
        _cache[key] = (x, {n: to_dev(a, w.dtype) for n, a in x.items()})
    return _cache[key]


def truncate(idx, cnt, processed):
    t = idx.copy()
    for u, c in np.ndenumerate(processed):
        t[u][c:] = -1
    return t, processed.astype(np.int32)


def check_processed(g, o, ratios, tau):
    diff = np.argwhere(g != o)
    for u in map(tuple, diff):
        d = min(int(g[u]), int(o[u])) - 1
        r = ratios[u][d]
        assert abs(r - tau) <= REL_TAU * max(tau, 1e-30), (u, int(g[u]), int(o[u]), r, tau)
    return len(diff)


def run(w, x, dev, idx, cnt, tau):
    out, _, proc = spa.spa_sparse_attn_prefill_early_stop(
        dev["q"], dev["k"], dev["v"], w.block, torch.from_numpy(idx).cuda(),
        torch.from_numpy(cnt).cuda(), w.scale, tau, w.n_sink, w.n_local)
    torch.cuda.synchronize()
    return to_host(out), proc.cpu().numpy()


def test_score_order_lists_match_oracle():
    w = PARITY_WORKLOADS["p_bf16_blk128"].with_(top_p=0.5)
    x, dev = inputs(w)
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    oidx, ocnt = oracle.score_order(sel, w.T, w.T, w.block, w.n_sink, w.n_local)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    gidx, gcnt = spa.spa_select_score_order(dev["q"], mean, var, w.block, w.scale, w.top_p,
                                            w.n_sink, w.n_local, w.k_min)
    torch.cuda.synchronize()
    gidx, gcnt = gidx.cpu().numpy(), gcnt.cpu().numpy()
    # same kept sets as the plain selection (near ties excused as there) ...
    srt = np.sort(np.where(np.arange(gidx.shape[-1]) < gcnt[..., None], gidx, 1 << 30), axis=-1)
    r = compare_lists(srt, gcnt, sel["idx"], sel["count"], sel["scores"], w.top_p, w.n_sink,
                      w.n_local, w.T, w.T, w.block)
    assert not r["unexcused"], r["unexcused"][:3]
    # ... in the oracle's traversal order wherever the sets agree
    for u, c in np.ndenumerate(gcnt):
        if c == ocnt[u] and set(gidx[u][:c]) == set(oidx[u][:c]):
            assert np.array_equal(gidx[u][:c], oidx[u][:c]), (u, gidx[u][:c], oidx[u][:c])
    assert spa.spa_get_device_error() == 0


@pytest.mark.parametrize("tau", [0.0, 0.02, 0.1, 0.3, 1.5])
def test_early_stop_matches_oracle(tau):
    w = PARITY_WORKLOADS["p_bf16_blk128"].with_(top_p=0.9)
    x, dev = inputs(w)
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    idx, cnt = oracle.score_order(sel, w.T, w.T, w.block, w.n_sink, w.n_local)
    g_out, g_proc = run(w, x, dev, idx, cnt, tau)
    o_proc, ratios = oracle.early_stop(x["q"], x["k"], w.dtype, w.block, idx, cnt, w.scale, tau,
                                       w.n_sink, w.n_local)
    nd = check_processed(g_proc, o_proc, ratios, tau)
    tidx, tcnt = truncate(idx, cnt, g_proc)
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, tidx, tcnt, w.scale)
    err = float(np.abs(g_out - o_out).max())
    print(f"\ntau {tau}: processed {g_proc.sum()} of {cnt.sum()} entries, {nd} excused "
          f"differences, max-abs {err:.3e}")
    assert err <= TOL
    if tau == 0.0:
        assert np.array_equal(g_proc, cnt)
    assert spa.spa_get_device_error() == 0


def test_early_stop_longer_lists():
    # 32 query blocks, one kv-group: lists long enough for the stop to bite
    w = PARITY_WORKLOADS["p_bf16_blk128"].with_(B=1, Hq=4, Hkv=1, T=4096, top_p=0.95)
    x, dev = inputs(w)
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    idx, cnt = oracle.score_order(sel, w.T, w.T, w.block, w.n_sink, w.n_local)
    for tau in (0.05, 0.2):
        g_out, g_proc = run(w, x, dev, idx, cnt, tau)
        o_proc, ratios = oracle.early_stop(x["q"], x["k"], w.dtype, w.block, idx, cnt, w.scale,
                                           tau, w.n_sink, w.n_local)
        nd = check_processed(g_proc, o_proc, ratios, tau)
        tidx, tcnt = truncate(idx, cnt, g_proc)
        o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, tidx, tcnt, w.scale)
        err = float(np.abs(g_out - o_out).max())
        print(f"\ntau {tau}: processed {g_proc.sum()} of {cnt.sum()} entries "
              f"({g_proc.sum() / cnt.sum():.3f}), {nd} excused, max-abs {err:.3e}")
        assert err <= TOL
        if tau == 0.2:
            # every row must agree before a query block stops, and the blocks are
            # ranked for the pooled query, not for each row: stops need a larger tau
            assert g_proc.sum() < cnt.sum()
    assert spa.spa_get_device_error() == 0


def test_early_stop_skips_repeats_and_out_of_range_entries():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, dev = inputs(w)
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    idx, cnt = oracle.score_order(sel, w.T, w.T, w.block, w.n_sink, w.n_local)
    bad = np.full(idx.shape[:-1] + (idx.shape[-1] + 4,), -1, np.int32)   # room for extra entries
    bad[..., :idx.shape[-1]] = idx
    bcnt = cnt.copy()
    u = (1, 3, 6)
    c = int(cnt[u])
    bad[u][:c + 2] = np.concatenate([idx[u][:2], [idx[u][0], w.nb + 4], idx[u][2:c]])
    bcnt[u] = c + 2
    g_out, g_proc = run(w, x, dev, bad, bcnt, 0.0)
    assert spa.spa_get_device_error() == 1          # SPA_DEVERR_BAD_INDEX
    assert g_proc[u] == c                           # the valid entries, once each
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, idx, cnt, w.scale)
    assert float(np.abs(g_out - o_out).max()) <= TOL
