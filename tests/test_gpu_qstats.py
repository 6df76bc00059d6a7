"""Parity of the quantised block statistics ("SpotAttention", section 4; INT4 and
FP4 (E2M1) microscale as read, format in include/spa.h) with the CPU oracle.

The quantiser is checked against the oracle's codes: they must be equal except in
groups where the oracle flags its own decision as a near tie (a value within 1e-5
relative of a half step, or the group maximum within 1e-5 of a scale boundary),
since the GPU's fp32 statistics differ from the oracle's in rounding order. The
selection on quantised statistics is checked on the oracle's own records, so its
kept lists must be bit-exact up to the usual excused near ties of the scores.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_stats_b200 as spa
from tests._parity import (compare_lists, pack_qstats, quant_ambiguous, to_dev, unpack_qstats)
from workloads import PARITY_WORKLOADS, WORKLOADS, generate

pytestmark = pytest.mark.gpu

_cache = {}


def inputs(w):
    key = (w.name, w.T, w.B, w.block, w.Hq, w.Hkv)
    if key not in _cache:
        x = generate(w)
        _cache.clear()
        _cache[key] = (x, {n: to_dev(a, w.dtype) for n, a in x.items()})
    return _cache[key]


FMTS = ["int4", "fp4"]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("key", list(PARITY_WORKLOADS))
def test_quantizer_matches_oracle_codes(key, fmt):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    rec = spa.spa_quantize_block_stats(mean, var, w.T, w.block, fmt=fmt)
    torch.cuda.synchronize()
    g = unpack_qstats(rec.cpu().numpy(), w.d, fmt)
    om, ov = oracle.block_stats(x["k"], w.dtype, w.block)
    o = oracle.quantize_stats(om, ov, fmt)
    amb = quant_ambiguous(om, ov, o)
    grp = lambda a: a.reshape(a.shape[:-1] + (w.d // 32, 32))
    diff = ((grp(g["cm"]) != grp(o["cm"])).any(-1) | (grp(g["cv"]) != grp(o["cv"])).any(-1) |
            (g["km"] != o["km"]) | (g["kv"] != o["kv"]))
    print(f"\n{w.name} {fmt}: {int(diff.sum())} of {diff.size} groups differ, "
          f"{int(amb.sum())} near ties flagged")
    assert not (diff & ~amb).any()
    assert rec.numel() == spa.spa_quantized_stats_bytes(w.B, w.Hkv, w.T, w.d, w.block)


@pytest.mark.parametrize("fmt", FMTS)
def test_quantizer_range_leaves_others_untouched(fmt):
    w = PARITY_WORKLOADS["d_bf16_blk16"]
    x, dev = inputs(w)
    mean, var = spa.spa_block_stats(dev["k"], w.block)
    rec = torch.full((w.B, w.Hkv, w.nb, w.d + w.d // 16), 0xAB, device="cuda", dtype=torch.uint8)
    spa.spa_quantize_block_stats(mean, var, w.T, w.block, w.nb - 3, w.nb, qstats=rec, fmt=fmt)
    torch.cuda.synchronize()
    r = rec.cpu().numpy()
    assert np.all(r[:, :, :w.nb - 3] == 0xAB)
    full = spa.spa_quantize_block_stats(mean, var, w.T, w.block, fmt=fmt).cpu().numpy()
    assert np.array_equal(r[:, :, w.nb - 3:], full[:, :, w.nb - 3:])


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("key", ["d_bf16_blk16", "d_bf16_blk64", "p_f32_d64", "p_bf16_blk128"])
def test_fused_stats_and_records_of_a_block_range(key, fmt):
    # spa_block_stats_quantized on the last blocks (a decode step's update): its
    # statistics match the oracle's, its records are exactly the oracle's quantiser
    # applied to those fp32 statistics, and blocks outside the range are untouched
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    nb = w.nb
    lo = max(0, nb - 3)
    mean = torch.full((w.B, w.Hkv, nb, w.d), 7.0, device="cuda")
    var = torch.full_like(mean, 7.0)
    rec = torch.full((w.B, w.Hkv, nb, w.d + w.d // 16), 0xAB, device="cuda", dtype=torch.uint8)
    spa.spa_block_stats_quantized(dev["k"], w.block, lo, nb, mean, var, rec, fmt=fmt)
    torch.cuda.synchronize()
    om, ov = oracle.block_stats(x["k"], w.dtype, w.block)
    m, v, r = mean.cpu().numpy(), var.cpu().numpy(), rec.cpu().numpy()
    np.testing.assert_allclose(m[:, :, lo:], om[:, :, lo:], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(v[:, :, lo:], ov[:, :, lo:], rtol=1e-5, atol=1e-6)
    assert np.all(m[:, :, :lo] == 7.0) and np.all(r[:, :, :lo] == 0xAB)
    o = oracle.quantize_stats(m[:, :, lo:].astype(np.float64), v[:, :, lo:].astype(np.float64), fmt)
    assert np.array_equal(r[:, :, lo:], pack_qstats(o))
    assert spa.spa_get_device_error() == 0


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("key", list(PARITY_WORKLOADS))
def test_select_quantized_on_oracle_records(key, fmt):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    sel = oracle.select_quantized(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink,
                                  w.n_local, w.k_min, fmt)
    rec = torch.from_numpy(pack_qstats(sel["q"])).cuda()
    idx, cnt = spa.spa_select_quantized(dev["q"], rec, w.T, w.block, w.scale, w.top_p, w.n_sink,
                                        w.n_local, w.k_min, fmt=fmt)
    torch.cuda.synchronize()
    r = compare_lists(idx.cpu().numpy(), cnt.cpu().numpy(), sel["idx"], sel["count"],
                      sel["scores"], w.top_p, w.n_sink, w.n_local, w.Lq, w.T, w.block)
    print(f"\n{w.name}: {r['units']} lists, {r['equal']} equal, {r['excused']} excused")
    assert not r["unexcused"], r["unexcused"][:3]
    assert spa.spa_get_device_error() == 0


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (8, 1), (16, 2)])
def test_select_quantized_decode_head_groupings(Hq, Hkv, fmt):
    # decode scoring on records runs on the tensor cores with the group's heads as
    # the MMA columns: one, two, eight (all columns) and eight heads per kv-head
    # (the four-head case is the parity workload above); a ragged candidate tile
    w = PARITY_WORKLOADS["d_bf16_blk16"].with_(Hq=Hq, Hkv=Hkv, T=16 * 300 + 5)
    x, dev = inputs(w)
    sel = oracle.select_quantized(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink,
                                  w.n_local, w.k_min, fmt)
    rec = torch.from_numpy(pack_qstats(sel["q"])).cuda()
    idx, cnt = spa.spa_select_quantized(dev["q"], rec, w.T, w.block, w.scale, w.top_p, w.n_sink,
                                        w.n_local, w.k_min, fmt=fmt)
    torch.cuda.synchronize()
    r = compare_lists(idx.cpu().numpy(), cnt.cpu().numpy(), sel["idx"], sel["count"],
                      sel["scores"], w.top_p, w.n_sink, w.n_local, w.Lq, w.T, w.block)
    print(f"\nG={Hq // Hkv}: {r['units']} lists, {r['equal']} equal, {r['excused']} excused")
    assert not r["unexcused"], r["unexcused"][:3]
    assert spa.spa_get_device_error() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_select_quantized_rule_variants(fmt):
    w = PARITY_WORKLOADS["d_bf16_blk16"]
    x, dev = inputs(w)
    for top_p, k_min in ((0.3, 0), (0.5, 20), (1.0, 0)):
        sel = oracle.select_quantized(x["q"], x["k"], w.dtype, w.block, w.scale, top_p, w.n_sink,
                                      w.n_local, k_min, fmt)
        rec = torch.from_numpy(pack_qstats(sel["q"])).cuda()
        idx, cnt = spa.spa_select_quantized(dev["q"], rec, w.T, w.block, w.scale, top_p,
                                            w.n_sink, w.n_local, k_min, fmt=fmt)
        torch.cuda.synchronize()
        r = compare_lists(idx.cpu().numpy(), cnt.cpu().numpy(), sel["idx"], sel["count"],
                          sel["scores"], top_p, w.n_sink, w.n_local, 1, w.T, w.block)
        assert not r["unexcused"], (top_p, k_min, r["unexcused"][:3])


@pytest.mark.slow
@pytest.mark.parametrize("fmt", FMTS)
def test_select_quantized_decode_workload_full_size(fmt):
    w = WORKLOADS[5]
    x = generate(w)
    q = to_dev(x["q"], w.dtype)
    sel = oracle.select_quantized(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, fmt=fmt)
    rec = torch.from_numpy(pack_qstats(sel["q"])).cuda()
    idx, cnt = spa.spa_select_quantized(q, rec, w.T, w.block, w.scale, w.top_p, fmt=fmt)
    torch.cuda.synchronize()
    r = compare_lists(idx.cpu().numpy(), cnt.cpu().numpy(), sel["idx"], sel["count"],
                      sel["scores"], w.top_p, w.n_sink, w.n_local, 1, w.T, w.block)
    plain = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p)
    overlap = []
    for u, c in np.ndenumerate(plain["count"]):
        a_, b_ = set(plain["idx"][u][:c].tolist()), set(sel["idx"][u][:sel["count"][u]].tolist())
        overlap.append(len(a_ & b_) / len(a_ | b_))
    print(f"\n{w.name} {fmt}: {r['units']} lists, {r['equal']} equal, {r['excused']} excused; "
          f"kept fraction {sel['count'].mean() / w.nb:.3f} (fp32 statistics "
          f"{plain['count'].mean() / w.nb:.3f}); mean Jaccard overlap with the fp32 "
          f"selection {np.mean(overlap):.4f}")
    assert not r["unexcused"], r["unexcused"][:3]
    assert spa.spa_get_device_error() == 0
