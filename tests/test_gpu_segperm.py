"""Parity of the segmented key permutation ("Sparsere Blok-Sparse Attention via
Tokenpermutatie", sections 2-3) with the CPU oracle.

The permutation is an order decided by floating point (fp32 importance on the
GPU, fp64 in the oracle): the GPU's permutation must keep each segment's keys and
be sorted by the oracle's importance except where two importances lie within
IMP_TOL (relative) of each other. The GPU's logits are exact bf16 products summed
in fp32; with |s q.k| up to about 30 on these inputs their rounding is up to a few
1e-5 absolute, which the exponential turns into relative errors of the same size
in a softmax weight. Selection and attention are checked on the oracle's own
permutation (the GPU gathers the permuted K/V from it): kept lists bit-exact up to
the usual excused near ties, outputs within 2e-2.
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
# segments of 256, 384 (ragged last) and 256 keys sort in registers; 24 blocks of
# 128 (3072 keys, one segment over the whole sequence) take the shared-memory sort
CASES = [("p_bf16_blk128", 2), ("p_bf16_blk128", 3), ("p_bf16_blk64", 4), ("p_bf16_blk128", 24)]

_cache = {}


def inputs(w):
    key = (w.name, w.T, w.B, w.block, w.Hq, w.Hkv)
    if key not in _cache:
        x = generate(w)
        _cache.clear()
        _cache[key] = (x, {n: to_dev(a, w.dtype) for n, a in x.items()})
    return _cache[key]


IMP_TOL = 1e-4


@pytest.mark.parametrize("key,seg", CASES)
def test_permutation_sorted_by_oracle_importance(key, seg):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    perm = spa.spa_pbs_permutation(dev["q"], dev["k"], w.block, seg, w.scale).cpu().numpy()
    operm, imp = oracle.pbs_permutation(x["q"], x["k"], w.dtype, w.block, seg, w.scale,
                                        return_importance=True)
    S = seg * w.block
    for b in range(w.B):
        for g in range(w.Hkv):
            for s0 in range(0, w.T, S):
                p = perm[b, g, s0:s0 + S]
                assert sorted(p.tolist()) == list(range(s0, min(s0 + S, w.T)))
                a = imp[b, g, p]
                worse = a[1:] > a[:-1] + IMP_TOL * np.maximum(np.abs(a[1:]), 1e-30)
                assert not worse.any(), (b, g, s0, np.flatnonzero(worse)[:3])
    print(f"\n{w.name} seg {seg}: {int((perm != operm).sum())} of {perm.size} positions differ "
          f"from the oracle's (near ties)")


def test_permutation_follows_the_softmax_weights_not_the_pooled_logit():
    # The hand-worked case of the oracle pins (rows 2, 3 of a 4-token sequence),
    # padded to d = 64 with zeros: the kernel must give the softmax-weight order
    # 2, 1, 0, 3 (the pooled logit would give 1, 0, 2, 3).
    import json, os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "worked_examples.json")))["segmented_permutation"]
    q = np.zeros((1, 1, 4, 64), np.float32)
    k = np.zeros((1, 1, 4, 64), np.float32)
    q[0, 0, :, :3] = g["q"]
    k[0, 0, :, :3] = g["k"]
    for dt in (torch.float32, torch.bfloat16):
        perm = spa.spa_pbs_permutation(torch.from_numpy(q).cuda().to(dt), torch.from_numpy(k).cuda().to(dt),
                                       g["block"], g["seg_blocks"], g["scale"])
        torch.cuda.synchronize()
        assert perm.cpu().numpy().reshape(-1).tolist() == g["expected_perm"]


def test_gather_is_exact():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, dev = inputs(w)
    operm = oracle.pbs_permutation(x["q"], x["k"], w.dtype, w.block, 2, w.scale)
    kp = spa.spa_pbs_gather(dev["k"], torch.from_numpy(operm).cuda())
    torch.cuda.synchronize()
    ref = oracle.permute(x["k"], operm)
    assert np.array_equal(kp.cpu().view(torch.int16).numpy().view(np.uint16), ref)


def segperm_setup(w, x, dev, seg, top_p):
    operm = oracle.pbs_permutation(x["q"], x["k"], w.dtype, w.block, seg, w.scale)
    pt = torch.from_numpy(operm).cuda()
    kp, vp = spa.spa_pbs_gather(dev["k"], pt), spa.spa_pbs_gather(dev["v"], pt)
    sel = oracle.select_segperm(x["q"], x["k"], w.dtype, w.block, seg, w.scale, top_p, w.n_sink,
                                w.n_local, w.k_min, perm=operm)
    return operm, kp, vp, sel


@pytest.mark.parametrize("key,seg", CASES)
def test_select_segperm_matches_oracle(key, seg):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    for top_p in (w.top_p, 0.5):
        operm, kp, vp, sel = segperm_setup(w, x, dev, seg, top_p)
        mean, var = spa.spa_block_stats(dev["k"], w.block)
        mp, vp_ = spa.spa_block_stats(kp, w.block)
        idx, cnt = spa.spa_select_segperm(dev["q"], mean, var, mp, vp_, w.block, seg, w.scale,
                                          top_p, w.n_sink, w.n_local, w.k_min)
        torch.cuda.synchronize()
        r = compare_lists(idx.cpu().numpy(), cnt.cpu().numpy(), sel["idx"], sel["count"],
                          sel["scores"], top_p, w.n_sink, w.n_local, w.T, w.T, w.block)
        print(f"\n{w.name} seg {seg} p {top_p}: {r['units']} lists, {r['equal']} equal, "
              f"{r['excused']} excused")
        assert not r["unexcused"], r["unexcused"][:3]
    assert spa.spa_get_device_error() == 0


@pytest.mark.parametrize("key,seg", CASES)
def test_attention_segperm_matches_oracle(key, seg):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    operm, kp, vp, sel = segperm_setup(w, x, dev, seg, 0.5)
    out, _ = spa.spa_sparse_attn_prefill_segperm(dev["q"], dev["k"], dev["v"], kp, vp, w.block,
                                                 seg, torch.from_numpy(sel["idx"]).cuda(),
                                                 torch.from_numpy(sel["count"]).cuda(), w.scale)
    torch.cuda.synchronize()
    o_out, _ = oracle.attention_segperm(x["q"], x["k"], x["v"], w.dtype, w.block, seg, operm,
                                        sel["idx"], sel["count"], w.scale)
    err = float(np.abs(to_host(out) - o_out).max())
    print(f"\n{w.name} seg {seg}: max-abs {err:.3e}")
    assert err <= TOL
    assert spa.spa_get_device_error() == 0


def test_attention_segperm_full_lists_are_dense_causal():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, dev = inputs(w)
    operm, kp, vp, _ = segperm_setup(w, x, dev, 3, 0.5)
    idx, cnt = oracle.full_lists(w.B, w.Hq, w.T, w.T, w.block)
    out, _ = spa.spa_sparse_attn_prefill_segperm(dev["q"], dev["k"], dev["v"], kp, vp, w.block, 3,
                                                 torch.from_numpy(idx).cuda(),
                                                 torch.from_numpy(cnt).cuda(), w.scale)
    torch.cuda.synchronize()
    dense, _ = oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, idx, cnt, w.scale)
    assert float(np.abs(to_host(out) - dense).max()) <= TOL
