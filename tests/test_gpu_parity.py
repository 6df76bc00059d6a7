"""Parity of the CUDA path (through the C-ABI) with the CPU oracle.

Tolerances: kept lists bit-exact except excused near ties (counted); attention
outputs max-abs 2e-2 for bf16 and 1e-4 for fp32; block statistics relative 1e-5.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_stats_b200 as spa
from tests._parity import compare_lists, sample_rows, to_dev, to_host
from workloads import PARITY_WORKLOADS, WORKLOADS, bf16_bits, generate, widen

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-2, "f32": 1e-4}
LSE_TOL = {"bf16": 2e-3, "f32": 1e-4}
PREFILL = [k for k, w in PARITY_WORKLOADS.items() if w.mode == "prefill"]
DECODE = [k for k, w in PARITY_WORKLOADS.items() if w.mode == "decode"]

_cache = {}


def inputs(w):
    key = (w.name, w.T, w.B, w.block, w.Hq, w.Hkv)  # the data depend on these only
    if key not in _cache:
        x = generate(w)
        _cache.clear()
        _cache[key] = (x, {n: to_dev(a, w.dtype) for n, a in x.items()})
    return _cache[key]


def oracle_select(w, x):
    return oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink,
                         w.n_local, w.k_min)


def assert_no_device_error():
    assert spa.spa_get_device_error() == 0


def check_lists(w, g_idx, g_cnt, sel, Lq):
    r = compare_lists(g_idx.cpu().numpy(), g_cnt.cpu().numpy(), sel["idx"], sel["count"],
                      sel["scores"], w.top_p, w.n_sink, w.n_local, Lq, w.T, w.block)
    print(f"\n{w.name}: {r['units']} lists, {r['equal']} equal, {r['excused']} excused near ties")
    assert not r["unexcused"], r["unexcused"][:3]
    return r


# ------------------------------------------------------------------ block statistics

@pytest.mark.parametrize("key", list(PARITY_WORKLOADS))
def test_block_stats_match_oracle(key):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    torch.cuda.synchronize()
    om, ov = oracle.block_stats(x["k"], w.dtype, w.block)
    np.testing.assert_allclose(mean.cpu().numpy(), om, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(var.cpu().numpy(), ov, rtol=1e-5, atol=1e-6)
    assert_no_device_error()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [16, 32, 64, 128])
def test_block_stats_every_shape_ragged_and_offset(dtype, d, block):
    # every (dtype, d, block) kernel shape; a ragged last block (1 row, and a
    # partial chunk), and keys 40 units off zero so that a merge of per-chunk
    # moments that cancelled badly would miss the variance tolerance
    rng = np.random.default_rng(1000 * block + d + (dtype == "bf16"))
    for T in (7 * block + 1, 5 * block + block // 2 + 3):
        k = 40.0 + rng.standard_normal((2, 3, T, d)) * rng.uniform(0.1, 2.0, (1, 3, 1, d))
        x = bf16_bits(k) if dtype == "bf16" else k.astype(np.float32)
        mean, var = spa.spa_block_stats(to_dev(x, dtype), block)
        torch.cuda.synchronize()
        om, ov = oracle.block_stats(x, dtype, block)
        np.testing.assert_allclose(mean.cpu().numpy(), om, rtol=1e-5, atol=1e-6)
        np.testing.assert_allclose(var.cpu().numpy(), ov, rtol=1e-5, atol=1e-6)
    assert_no_device_error()


def test_block_stats_incremental_range_touches_only_its_blocks():
    w = PARITY_WORKLOADS["d_bf16_blk16"]
    x, dev = inputs(w)
    full_m, full_v = spa.spa_block_stats(dev["k"], w.block)
    m = torch.full_like(full_m, 7.0)
    v = torch.full_like(full_v, 7.0)
    nb = w.nb
    spa.spa_block_stats(dev["k"], w.block, nb - 3, nb, mean=m, var=v)
    torch.cuda.synchronize()
    assert torch.equal(m[:, :, nb - 3:], full_m[:, :, nb - 3:])
    assert torch.equal(v[:, :, nb - 3:], full_v[:, :, nb - 3:])
    assert torch.all(m[:, :, :nb - 3] == 7.0) and torch.all(v[:, :, :nb - 3] == 7.0)


# ------------------------------------------------------------------ selection

@pytest.mark.parametrize("key", list(PARITY_WORKLOADS))
def test_select_matches_oracle(key):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    idx, cnt = spa.spa_select(dev["q"], mean, var, w.T, w.block, w.scale, w.top_p, w.n_sink,
                              w.n_local, w.k_min)
    torch.cuda.synchronize()
    check_lists(w, idx, cnt, oracle_select(w, x), w.Lq)
    assert_no_device_error()


@pytest.mark.parametrize("p,k_min,n_sink,n_local", [(1.0, 0, 1, 1), (1e-4, 0, 1, 1),
                                                   (0.5, 3, 2, 2), (0.7, 0, 0, 0)])
def test_select_rule_variants(p, k_min, n_sink, n_local):
    w = PARITY_WORKLOADS["p_bf16_blk64"].with_(top_p=p, k_min=k_min, n_sink=n_sink,
                                                 n_local=n_local)
    x, dev = inputs(w)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    idx, cnt = spa.spa_select(dev["q"], mean, var, w.T, w.block, w.scale, p, n_sink, n_local,
                              k_min)
    torch.cuda.synchronize()
    check_lists(w, idx, cnt, oracle_select(w, x), w.Lq)


# ------------------------------------------------------------------ attention

@pytest.mark.parametrize("key", PREFILL)
def test_prefill_matches_oracle_on_oracle_lists(key):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    sel = oracle_select(w, x)
    idx = torch.from_numpy(sel["idx"]).cuda()
    cnt = torch.from_numpy(sel["count"]).cuda()
    out, lse = spa.spa_sparse_attn_prefill(dev["q"], dev["k"], dev["v"], w.block, idx, cnt,
                                           w.scale, want_lse=True)
    torch.cuda.synchronize()
    o_out, o_lse = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                    sel["count"], w.scale)
    err = np.abs(to_host(out) - o_out).max()
    print(f"\n{w.name}: max-abs {err:.3e}")
    assert err <= TOL[w.dtype]
    np.testing.assert_allclose(lse.cpu().numpy(), o_lse, rtol=0, atol=LSE_TOL[w.dtype])
    assert_no_device_error()


@pytest.mark.parametrize("key", PREFILL)
def test_prefill_pipeline_matches_oracle(key):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    r = spa.prefill(dev["q"], dev["k"], dev["v"], w.block, w.top_p, w.scale, w.n_sink, w.n_local,
                    w.k_min)
    torch.cuda.synchronize()
    sel = oracle_select(w, x)
    check_lists(w, r["idx"], r["count"], sel, w.Lq)
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                sel["count"], w.scale)
    g_cnt = r["count"].cpu().numpy()
    g_idx = r["idx"].cpu().numpy()
    out = to_host(r["out"])
    for b in range(w.B):
        for h in range(w.Hq):
            for i in range(w.nq):
                c = g_cnt[b, h, i]
                if c == sel["count"][b, h, i] and np.array_equal(g_idx[b, h, i, :c],
                                                                  sel["idx"][b, h, i, :c]):
                    rows = slice(i * w.block, min(w.T, (i + 1) * w.block))
                    assert np.abs(out[b, h, rows] - o_out[b, h, rows]).max() <= TOL[w.dtype]


def test_prefill_top_p_one_is_dense_causal_attention():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, dev = inputs(w)
    r = spa.prefill(dev["q"], dev["k"], dev["v"], w.block, 1.0, w.scale)
    torch.cuda.synchronize()
    fi, fc = oracle.full_lists(w.B, w.Hq, w.T, w.T, w.block)
    assert np.array_equal(r["count"].cpu().numpy(), fc)
    dense, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, fi, fc, w.scale)
    assert np.abs(to_host(r["out"]) - dense).max() <= TOL[w.dtype]


@pytest.mark.parametrize("L,block", [(64, 128), (128, 128), (130, 128), (200, 64), (64, 64),
                                     (40, 64)])
def test_prefill_short_and_ragged_sequences(L, block):
    w = PARITY_WORKLOADS["p_bf16_blk128"].with_(T=L, block=block, B=1)
    x, dev = inputs(w)
    r = spa.prefill(dev["q"], dev["k"], dev["v"], w.block, w.top_p, w.scale)
    torch.cuda.synchronize()
    sel = oracle_select(w, x)
    check_lists(w, r["idx"], r["count"], sel, w.Lq)
    idx = torch.from_numpy(sel["idx"]).cuda()
    cnt = torch.from_numpy(sel["count"]).cuda()
    out, _ = spa.spa_sparse_attn_prefill(dev["q"], dev["k"], dev["v"], w.block, idx, cnt, w.scale)
    torch.cuda.synchronize()
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                sel["count"], w.scale)
    assert np.abs(to_host(out) - o_out).max() <= TOL[w.dtype]


@pytest.mark.parametrize("key", DECODE)
def test_decode_matches_oracle(key):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    sel = oracle_select(w, x)
    idx = torch.from_numpy(sel["idx"]).cuda()
    cnt = torch.from_numpy(sel["count"]).cuda()
    out = spa.spa_sparse_attn_decode(dev["q"], dev["k"], dev["v"], w.block, idx, cnt, w.scale)
    torch.cuda.synchronize()
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                sel["count"], w.scale)
    err = np.abs(to_host(out) - o_out).max()
    print(f"\n{w.name}: max-abs {err:.3e}")
    assert err <= TOL[w.dtype]
    # the whole decode step through the binding
    r = spa.decode(dev["q"], dev["k"], dev["v"], w.block, w.top_p, scale=w.scale)
    torch.cuda.synchronize()
    check_lists(w, r["idx"], r["count"], sel, 1)
    assert_no_device_error()


@pytest.mark.parametrize("Hq,Hkv,block,T", [(2, 2, 16, 1000), (8, 1, 32, 777), (16, 1, 128, 1500),
                                            (6, 2, 64, 3000), (16, 2, 16, 129)])
def test_decode_random_lists_groupings_and_edges(Hq, Hkv, block, T):
    # Lists the selection would never write: random subsets, an empty list (the
    # output is zero, as the oracle's), every block, the sink alone, the last block
    # alone; G = 1, 3, 8 and 16 query heads per kv-head; ragged and one-token tails.
    w = PARITY_WORKLOADS["d_bf16_blk16"].with_(Hq=Hq, Hkv=Hkv, block=block, T=T, B=2)
    x, dev = inputs(w)
    rng = np.random.default_rng(Hq * 1000 + block)
    idx = np.full((w.B, w.Hq, 1, w.nb), -1, np.int32)
    cnt = np.zeros((w.B, w.Hq, 1), np.int32)
    for b in range(w.B):
        for h in range(w.Hq):
            kind = (b * w.Hq + h) % 5
            if kind == 0:
                keep = []
            elif kind == 1:
                keep = list(range(w.nb))
            elif kind == 2:
                keep = [0]
            elif kind == 3:
                keep = [w.nb - 1]
            else:
                keep = [j for j in range(w.nb) if rng.random() < 0.3]
            idx[b, h, 0, :len(keep)] = keep
            cnt[b, h, 0] = len(keep)
    out = spa.spa_sparse_attn_decode(dev["q"], dev["k"], dev["v"], w.block,
                                     torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                                     w.scale)
    torch.cuda.synchronize()
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, idx, cnt, w.scale)
    g = to_host(out)
    assert np.abs(g - o_out).max() <= TOL[w.dtype]
    empty = cnt[:, :, 0] == 0
    assert (g[empty] == 0).all()
    assert_no_device_error()


def _prefill_matches_oracle(w, x, dev):
    sel = oracle_select(w, x)
    out, _ = spa.spa_sparse_attn_prefill(dev["q"], dev["k"], dev["v"], w.block,
                                         torch.from_numpy(sel["idx"]).cuda(),
                                         torch.from_numpy(sel["count"]).cuda(), w.scale)
    torch.cuda.synchronize()
    ref, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"], sel["count"],
                              w.scale)
    assert float(np.abs(to_host(out) - ref).max()) <= TOL[w.dtype]


def test_bounded_wait_runs_out_and_reports_timeout():
    # The failure path every kernel's waits share: a barrier that nothing completes.
    # The wait gives up after its limit, records the timeout in the device error
    # word, and the context stays usable for the next launch. The prefill kernel
    # (whose waits are the same bounded waits) runs correctly after it.
    assert spa.spa_get_device_error() == 0
    spa.spa_selftest_wait_timeout(2000)
    assert spa.spa_get_device_error() == 3      # SPA_DEVERR_TIMEOUT
    assert spa.spa_get_device_error() == 0      # reading clears it
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, dev = inputs(w)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    torch.cuda.synchronize()
    om, ov = oracle.block_stats(x["k"], w.dtype, w.block)
    np.testing.assert_allclose(mean.cpu().numpy(), om, rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(var.cpu().numpy(), ov, rtol=1e-5, atol=1e-6)
    _prefill_matches_oracle(w, x, dev)
    assert_no_device_error()


def test_timeout_ends_only_its_own_launch():
    # A launch after a timed-out one, before anybody read the error word, still
    # waits normally: giving up early is keyed to the launch that ran out. The code
    # itself stays set until it is read.
    assert spa.spa_get_device_error() == 0
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, dev = inputs(w)
    spa.spa_selftest_wait_timeout(2000)
    _prefill_matches_oracle(w, x, dev)
    assert spa.spa_get_device_error() == 3
    assert spa.spa_get_device_error() == 0


def _valid_entries(lst, i):
    """The list as the kernels walk it: an entry is kept when it lies in [0, i] and
    exceeds the last kept entry; the rest are skipped (and reported)."""
    out, last = [], -1
    for j in lst:
        if 0 <= j <= i and j > last:
            out.append(j)
            last = j
    return out


@pytest.mark.parametrize("key", ["p_bf16_blk128", "p_f32_d64"])
def test_corrupt_lists_are_reported_and_skipped(key):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    sel = oracle_select(w, x)
    idx = sel["idx"].copy()
    cnt = sel["count"].copy()
    idx[0, 0, 5, 1] = 7          # beyond the causal limit of query block 5: skipped
    idx[0, 1, 6, 2] = 0          # not ascending: skipped
    # a longer mix on the last query block: out of range, repeats, a step back
    last_i = w.nq - 1
    idx[0, 0, last_i, :8] = [0, 3, last_i + 40, 5, 5, 4, -3, 6]
    cnt[0, 0, last_i] = 8
    ref_idx, ref_cnt = np.full_like(idx, -1), cnt.copy()
    for u, c in np.ndenumerate(cnt):
        keep = _valid_entries(idx[u][:c].tolist(), u[2])
        ref_idx[u][:len(keep)] = keep
        ref_cnt[u] = len(keep)
    out, _ = spa.spa_sparse_attn_prefill(dev["q"], dev["k"], dev["v"], w.block,
                                         torch.from_numpy(idx).cuda(),
                                         torch.from_numpy(cnt).cuda(), w.scale)
    assert spa.spa_get_device_error() == 1      # SPA_DEVERR_BAD_INDEX
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, ref_idx, ref_cnt,
                                w.scale)
    assert np.abs(to_host(out) - o_out).max() <= TOL[w.dtype]
    cnt2 = sel["count"].copy()
    cnt2[w.B - 1, w.Hq - 1, 2] = w.nb + 5       # count beyond cap: clamped
    spa.spa_sparse_attn_prefill(dev["q"], dev["k"], dev["v"], w.block,
                                torch.from_numpy(sel["idx"]).cuda(),
                                torch.from_numpy(cnt2).cuda(), w.scale)
    assert spa.spa_get_device_error() == 2      # SPA_DEVERR_BAD_COUNT
    assert spa.spa_get_device_error() == 0      # reading clears it


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_block_stats_of_a_block_range_equal_the_full_launch(block, dtype):
    # a sub-range [blk_begin, blk_end) of blocks of 64+ keys (the one-warp-per-block
    # kernel) writes exactly what the full launch writes there, and nothing else
    rng = np.random.default_rng(block + (dtype == "bf16"))
    T = 9 * block + 17
    k = rng.standard_normal((2, 3, T, 128)) * 1.5 + 0.25
    kd = to_dev(bf16_bits(k) if dtype == "bf16" else k.astype(np.float32), dtype)
    full_m, full_v = spa.spa_block_stats(kd, block)
    nb = full_m.shape[2]
    m = torch.full_like(full_m, 7.0)
    v = torch.full_like(full_v, 7.0)
    spa.spa_block_stats(kd, block, 3, nb, mean=m, var=v)
    torch.cuda.synchronize()
    assert torch.equal(m[:, :, 3:], full_m[:, :, 3:]) and torch.equal(v[:, :, 3:], full_v[:, :, 3:])
    assert torch.all(m[:, :, :3] == 7.0) and torch.all(v[:, :, :3] == 7.0)


# ------------------------------------------------------------------ headline workloads

@pytest.mark.slow
def test_tiny_fp32_workload_full():
    w = WORKLOADS[1]
    x = generate(w)
    dev = {n: to_dev(a, w.dtype) for n, a in x.items()}
    r = spa.prefill(dev["q"], dev["k"], dev["v"], w.block, w.top_p, w.scale, want_lse=True)
    torch.cuda.synchronize()
    sel = oracle_select(w, x)
    check_lists(w, r["idx"], r["count"], sel, w.Lq)
    o_out, o_lse = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                    sel["count"], w.scale)
    assert np.abs(to_host(r["out"]) - o_out).max() <= TOL["f32"]
    assert np.abs(r["lse"].cpu().numpy() - o_lse).max() <= LSE_TOL["f32"]


@pytest.mark.slow
@pytest.mark.parametrize("cid", [2, 3, 4])
def test_prefill_workload_full_size(cid):
    w = WORKLOADS[cid]
    x = generate(w)
    dev = {n: to_dev(a, w.dtype) for n, a in x.items()}
    r = spa.prefill(dev["q"], dev["k"], dev["v"], w.block, w.top_p, w.scale)
    torch.cuda.synchronize()
    sel = oracle_select(w, x)
    res = check_lists(w, r["idx"], r["count"], sel, w.Lq)
    kept = sel["count"].sum() / (w.B * w.Hq * w.nq * (w.nq + 1) / 2)
    print(f"kept fraction of causal blocks: {kept:.3f}; excused {res['excused']}")
    # outputs on sampled rows, both through the kernel on the oracle's lists and
    # through the full pipeline where the lists agree
    idx = torch.from_numpy(sel["idx"]).cuda()
    cnt = torch.from_numpy(sel["count"]).cuda()
    out, _ = spa.spa_sparse_attn_prefill(dev["q"], dev["k"], dev["v"], w.block, idx, cnt, w.scale)
    torch.cuda.synchronize()
    rows = sample_rows(w.B, w.Hq, w.T, w.block, 96, cid)
    o_rows, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                 sel["count"], w.scale, rows=rows)
    g_rows = to_host(out.reshape(-1, w.d)[torch.from_numpy(rows).cuda()])
    err = np.abs(g_rows - o_rows).max()
    print(f"{w.name}: sampled max-abs {err:.3e}")
    assert err <= TOL[w.dtype]
    assert_no_device_error()


@pytest.mark.slow
def test_decode_workload_full_size():
    w = WORKLOADS[5]
    x = generate(w)
    dev = {n: to_dev(a, w.dtype) for n, a in x.items()}
    r = spa.decode(dev["q"], dev["k"], dev["v"], w.block, w.top_p, scale=w.scale)
    torch.cuda.synchronize()
    sel = oracle_select(w, x)
    res = check_lists(w, r["idx"], r["count"], sel, 1)
    print(f"kept fraction {sel['count'].mean() / w.nb:.3f}; excused {res['excused']}")
    idx = torch.from_numpy(sel["idx"]).cuda()
    cnt = torch.from_numpy(sel["count"]).cuda()
    out = spa.spa_sparse_attn_decode(dev["q"], dev["k"], dev["v"], w.block, idx, cnt, w.scale)
    torch.cuda.synchronize()
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                sel["count"], w.scale)
    err = np.abs(to_host(out) - o_out).max()
    print(f"{w.name}: max-abs {err:.3e}")
    assert err <= TOL[w.dtype]
    assert_no_device_error()


@pytest.mark.parametrize("T,Hq,Hkv", [(3000, 4, 1), (3000, 4, 2), (3000, 2, 2), (4000, 8, 1),
                                     (6000, 8, 2), (12000, 8, 2), (12000, 8, 1)])
def test_select_many_candidates(T, Hq, Hkv):
    # 188 and 250 blocks of 16: 129 to 256 residual candidates are sorted by a pair
    # of warps per head where the CTA has two warps per head (G = 1, 2, 4), by one
    # warp otherwise (G = 8); 375 and 750 blocks: more candidates than a warp pair
    # sorts, so the grouped kernel sorts each head across the CTA (2 and 4 keys per
    # thread)
    w = PARITY_WORKLOADS["p_bf16_blk128"].with_(T=T, B=1, Hq=Hq, Hkv=Hkv, block=16)
    x, dev = inputs(w)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    idx, cnt = spa.spa_select(dev["q"], mean, var, w.T, w.block, w.scale, w.top_p, w.n_sink,
                              w.n_local, w.k_min)
    torch.cuda.synchronize()
    sel = oracle_select(w, x)
    check_lists(w, idx, cnt, sel, w.Lq)
    # traversal order (the early-stop lists) from the same path
    gidx, gcnt = spa.spa_select_score_order(dev["q"], mean, var, w.block, w.scale, w.top_p,
                                            w.n_sink, w.n_local, w.k_min)
    torch.cuda.synchronize()
    oidx, ocnt = oracle.score_order(sel, w.T, w.T, w.block, w.n_sink, w.n_local)
    gidx, gcnt = gidx.cpu().numpy(), gcnt.cpu().numpy()
    same = ordered = 0
    for u, c in np.ndenumerate(gcnt):
        if c == ocnt[u] and set(gidx[u][:c]) == set(oidx[u][:c]):
            same += 1
            if np.array_equal(gidx[u][:c], oidx[u][:c]):
                ordered += 1
                continue
            # the residual part follows the oracle's scores, up to near ties (two
            # fp32 scores within rounding may come out in either order)
            i = u[-1]
            r_lo = min(w.n_sink, i + 1)
            r_hi = max(r_lo, i - w.n_local + 1)
            start = (i + 1 - r_hi) + r_lo
            sc = sel["scores"][u][gidx[u][start:c]]
            tol = 1e-5 * np.maximum(1.0, np.abs(sc[:-1]))
            assert np.all(sc[1:] <= sc[:-1] + tol), (u, gidx[u][start:c])
    print(f"{same} of {gcnt.size} sets equal, {ordered} in the identical order")
    assert same >= 0.9 * gcnt.size
    assert_no_device_error()


@pytest.mark.parametrize("Hq,Hkv,block,dtype", [(4, 4, 128, "bf16"), (4, 2, 128, "bf16"),
                                                (8, 2, 128, "bf16"), (8, 1, 64, "bf16"),
                                                (6, 2, 64, "bf16"), (8, 1, 64, "f32")])
def test_select_head_groupings(Hq, Hkv, block, dtype):
    # G = 1, 2, 4, 8 query heads per kv-head take the grouped selection kernel (one
    # CTA per kv-head and query block, a warp per head for the sort and cut); G = 3
    # takes the per-head kernel; the fp32 case reads fp32 queries
    base = "p_bf16_blk128" if dtype == "bf16" else "p_f32_d128"
    w = PARITY_WORKLOADS[base].with_(Hq=Hq, Hkv=Hkv, block=block, B=1, T=777)
    x, dev = inputs(w)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    idx, cnt = spa.spa_select(dev["q"], mean, var, w.T, w.block, w.scale, w.top_p, w.n_sink,
                              w.n_local, w.k_min)
    torch.cuda.synchronize()
    check_lists(w, idx, cnt, oracle_select(w, x), w.Lq)
    assert_no_device_error()


@pytest.mark.parametrize("Hq,Hkv,block", [(4, 4, 128), (4, 2, 128), (8, 2, 128), (2, 1, 64),
                                          (4, 1, 64), (8, 2, 64)])
def test_prefill_head_groupings(Hq, Hkv, block):
    # One, two or four query heads per kv-head: exercises the two-tile kernel (two
    # tiles of the same kv-group fit) and the single-tile kernel (they do not).
    w = PARITY_WORKLOADS["p_bf16_blk128"].with_(Hq=Hq, Hkv=Hkv, block=block, B=1, T=777)
    x, dev = inputs(w)
    sel = oracle_select(w, x)
    idx = torch.from_numpy(sel["idx"]).cuda()
    cnt = torch.from_numpy(sel["count"]).cuda()
    out, lse = spa.spa_sparse_attn_prefill(dev["q"], dev["k"], dev["v"], w.block, idx, cnt,
                                           w.scale, want_lse=True)
    torch.cuda.synchronize()
    o_out, o_lse = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"],
                                    sel["count"], w.scale)
    assert np.abs(to_host(out) - o_out).max() <= TOL[w.dtype]
    np.testing.assert_allclose(lse.cpu().numpy(), o_lse, rtol=0, atol=LSE_TOL[w.dtype])
    assert_no_device_error()


@pytest.mark.parametrize("outlier", [False, True])
def test_decode_cut_dense_bin(outlier):
    # every residual block with the same statistics: equal scores, so the cut falls
    # in a score bin of ~600 candidates (more than one warp sorts) and the exact
    # bisection decides; ties are kept in index order on both sides
    w = PARITY_WORKLOADS["d_bf16_blk16"].with_(T=16 * 600, B=1, top_p=0.9)
    x = generate(w)
    k = np.tile(x["k"][:, :, :w.block, :], (1, 1, w.T // w.block, 1))
    if outlier:   # one block well above the rest, still short of top_p alone
        q = widen(x["q"], w.dtype)
        G = w.Hq // w.Hkv
        for g in range(w.Hkv):
            k[0, g, 100 * w.block:101 * w.block, :] = bf16_bits(0.2 * q[0, g * G, -1, :])[None, :]
    x = dict(x, k=np.ascontiguousarray(k))
    dev = {n: to_dev(a, w.dtype) for n, a in x.items()}
    r = spa.decode(dev["q"], dev["k"], dev["v"], w.block, w.top_p, scale=w.scale, k_min=w.k_min)
    torch.cuda.synchronize()
    sel = oracle_select(w, x)
    res = check_lists(w, r["idx"], r["count"], sel, 1)
    assert res["equal"] == res["units"]
    assert_no_device_error()


@pytest.mark.parametrize("p,k_min", [(0.9, 0), (1e-4, 0), (0.3, 200), (1.0, 0), (0.999, 0)])
def test_decode_select_long_residual_rule_variants(p, k_min):
    # 1250 candidate blocks per head: the selection's wide (register-held) cut.
    w = PARITY_WORKLOADS["d_bf16_blk16"].with_(T=20000, B=2, top_p=p, k_min=k_min)
    x, dev = inputs(w)
    r = spa.decode(dev["q"], dev["k"], dev["v"], w.block, p, scale=w.scale, k_min=k_min)
    torch.cuda.synchronize()
    sel = oracle_select(w, x)
    check_lists(w, r["idx"], r["count"], sel, 1)
    o_out, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"], sel["count"],
                                w.scale)
    same = all(np.array_equal(r["idx"].cpu().numpy()[b, h, 0, :c], sel["idx"][b, h, 0, :c])
               for b in range(w.B) for h in range(w.Hq) for c in [sel["count"][b, h, 0]])
    if same:
        assert np.abs(to_host(r["out"]) - o_out).max() <= TOL[w.dtype]
    assert_no_device_error()
