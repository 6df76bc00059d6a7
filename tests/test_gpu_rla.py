"""Parity of the Residual Linear Attention kernels (through the C-ABI) with the CPU
oracle ("SPLA - Block Sparse Plus Linear Attention for Long Context Modeling",
sections 2.2-2.3).

Tolerance, derived from the arithmetic: the kernels round exp(k), exp(q), each
block state W_j and the masked scores of an unkept own block to bf16, whose unit
roundoff is u = 2^-8 (8-bit significand, round to nearest even), and accumulate in
fp32. A state W_j carries two roundings (exp(k), W_j); every branch output element
is a sum of products with three rounded factors (exp(q), exp(k), W_j; or exp(q),
exp(k), the rounded score). So |error| <= ((1 + u)^r - 1) * mag plus the fp32
accumulation error, where r is 2 or 3 and mag is the same sum taken with |v| (the
oracle's `mag`, or the state of |v|). The tests allow (r + 0.2) * u * mag.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_long_stats_b200 as spa
from tests._parity import sample_rows, to_dev, to_host
from workloads import PARITY_WORKLOADS, WORKLOADS, generate

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8
STATE_ROUNDINGS, OUTPUT_ROUNDINGS = 2, 3
PREFILL_BF16 = [k for k, w in PARITY_WORKLOADS.items() if w.mode == "prefill" and w.dtype == "bf16"]

_cache = {}


def inputs(w):
    key = (w.name, w.T, w.B, w.block, w.Hq, w.Hkv)
    if key not in _cache:
        x = generate(w)
        _cache.clear()
        _cache[key] = (x, {n: to_dev(a, w.dtype) for n, a in x.items()})
    return _cache[key]


def within(g, o, mag, what, roundings=OUTPUT_ROUNDINGS):
    """Checks |g - o| <= (roundings + 0.2) u mag elementwise; returns the worst
    |g - o| / mag."""
    rel = (roundings + 0.2) * U_BF16
    err = np.abs(g - o)
    bad = err > rel * mag + 1e-30
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} beyond {rel:.3e} * mag; "
                           f"worst ratio {float((err / np.maximum(mag, 1e-30)).max()):.3e}")
    return float((err / np.maximum(mag, 1e-30)).max())


def abs_v(x):
    """The same inputs with |v| (bf16 bit patterns: clear the sign bit)."""
    y = dict(x)
    y["v"] = x["v"] & np.uint16(0x7FFF)
    return y


def lists_without_own_block(w, seed):
    """Random ascending lists that may leave out the sink and the own block."""
    rng = np.random.default_rng(seed)
    idx = np.full((w.B, w.Hq, w.nq, w.nb), -1, np.int32)
    cnt = np.zeros((w.B, w.Hq, w.nq), np.int32)
    for b in range(w.B):
        for h in range(w.Hq):
            for i in range(w.nq):
                keep = [j for j in range(i + 1) if rng.random() < 0.6]
                idx[b, h, i, :len(keep)] = keep
                cnt[b, h, i] = len(keep)
    return idx, cnt


@pytest.mark.parametrize("key", PREFILL_BF16)
def test_block_states_match_oracle(key):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    st = spa.spa_rla_block_states(dev["k"], dev["v"], w.block)
    torch.cuda.synchronize()
    o = oracle.rla_block_states(x["k"], x["v"], "bf16", w.block)
    m = oracle.rla_block_states(x["k"], abs_v(x)["v"], "bf16", w.block)
    r = within(to_host(st), o, m, f"{w.name} states", STATE_ROUNDINGS)
    print(f"\n{w.name}: worst |err| / mag = {r:.3e}")
    assert spa.spa_get_device_error() == 0


def test_block_states_range_leaves_others_untouched():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, dev = inputs(w)
    st = torch.full((w.B, w.Hkv, w.nb, 128, 128), float("nan"), device="cuda", dtype=torch.bfloat16)
    spa.spa_rla_block_states(dev["k"], dev["v"], w.block, 2, 5, states=st)
    torch.cuda.synchronize()
    g = to_host(st)
    assert np.isnan(g[:, :, :2]).all() and np.isnan(g[:, :, 5:]).all()
    o = oracle.rla_block_states(x["k"], x["v"], "bf16", w.block)[:, :, 2:5]
    m = oracle.rla_block_states(x["k"], abs_v(x)["v"], "bf16", w.block)[:, :, 2:5]
    within(g[:, :, 2:5], o, m, "range", STATE_ROUNDINGS)


def run_rla(w, dev, idx, cnt):
    st = spa.spa_rla_block_states(dev["k"], dev["v"], w.block)
    out = spa.spa_rla_prefill(dev["q"], dev["k"], dev["v"], st, w.block,
                              torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda())
    torch.cuda.synchronize()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("top_p", [None, 0.3])
@pytest.mark.parametrize("key", PREFILL_BF16)
def test_rla_prefill_on_oracle_lists(key, top_p):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    if top_p is not None:                      # same data, a smaller nucleus: residual blocks
        w = w.with_(top_p=top_p)
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    g = run_rla(w, dev, sel["idx"], sel["count"])
    o, m = oracle.rla(x["q"], x["k"], x["v"], "bf16", w.block, sel["idx"], sel["count"])
    r = within(g, o, m, w.name)
    print(f"\n{w.name}: worst |err| / mag = {r:.3e}, residual rows {int((m > 0).any(-1).sum())}")
    assert spa.spa_get_device_error() == 0


@pytest.mark.parametrize("key", PREFILL_BF16)
def test_rla_prefill_own_block_left_out(key):
    # lists that drop the sink and the query's own block: the causal token path
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    idx, cnt = lists_without_own_block(w, 7)
    g = run_rla(w, dev, idx, cnt)
    o, m = oracle.rla(x["q"], x["k"], x["v"], "bf16", w.block, idx, cnt)
    r = within(g, o, m, w.name + " without own block")
    print(f"\n{w.name} without own block: worst |err| / mag = {r:.3e}")
    assert spa.spa_get_device_error() == 0


def test_rla_prefill_full_lists_give_zero_and_empty_lists_global():
    w = PARITY_WORKLOADS["p_bf16_blk64"]
    x, dev = inputs(w)
    idx, cnt = oracle.full_lists(w.B, w.Hq, w.T, w.T, w.block)
    g = run_rla(w, dev, idx, cnt)
    assert np.all(g == 0.0)
    cnt0 = np.zeros_like(cnt)                  # nothing kept: global causal linear attention
    g = run_rla(w, dev, idx, cnt0)
    rows = sample_rows(w.B, w.Hq, w.T, w.block, 64, 3)
    o, m = oracle.rla(x["q"], x["k"], x["v"], "bf16", w.block, idx, cnt0, rows=rows)
    within(g.reshape(-1, 128)[rows], o, m, "global")
    assert spa.spa_get_device_error() == 0


def test_rla_prefill_corrupt_lists_report_device_errors():
    w = PARITY_WORKLOADS["p_bf16_blk128"]
    x, dev = inputs(w)
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    idx, cnt = sel["idx"].copy(), sel["count"].copy()
    idx[0, 1, 5, 0] = w.nb + 3                  # out of range: skipped
    run_rla(w, dev, idx, cnt)
    assert spa.spa_get_device_error() == 1      # SPA_DEVERR_BAD_INDEX
    cnt2 = sel["count"].copy()
    cnt2[1, 2, 3] = -4                          # negative count: clamped to 0
    g = run_rla(w, dev, sel["idx"], cnt2)
    assert spa.spa_get_device_error() == 2      # SPA_DEVERR_BAD_COUNT
    cnt3 = sel["count"].copy()
    cnt3[1, 2, 3] = 0
    o, m = oracle.rla(x["q"], x["k"], x["v"], "bf16", w.block, sel["idx"], cnt3,
                      rows=np.arange(((1 * w.Hq + 2) * w.T + 3 * w.block),
                                     ((1 * w.Hq + 2) * w.T + 4 * w.block), dtype=np.int64))
    within(g[1, 2, 3 * w.block:4 * w.block], o, m, "clamped count")


@pytest.mark.slow
def test_rla_prefill_full_size_sampled_rows():
    w = WORKLOADS[3]
    x = generate(w)
    dev = {n: to_dev(a, w.dtype) for n, a in x.items()}
    r = spa.prefill(dev["q"], dev["k"], dev["v"], w.block, w.top_p, w.scale)
    st = spa.spa_rla_block_states(dev["k"], dev["v"], w.block)
    out = spa.spa_rla_prefill(dev["q"], dev["k"], dev["v"], st, w.block, r["idx"], r["count"])
    torch.cuda.synchronize()
    rows = sample_rows(w.B, w.Hq, w.T, w.block, 96, 11)
    g = out.reshape(-1, 128)[torch.from_numpy(rows).cuda()].cpu().numpy().astype(np.float64)
    o, m = oracle.rla(x["q"], x["k"], x["v"], "bf16", w.block, r["idx"].cpu().numpy(),
                      r["count"].cpu().numpy(), rows=rows)
    print(f"\n{w.name}: worst |err| / mag = {within(g, o, m, w.name):.3e}")
    assert spa.spa_get_device_error() == 0


# ------------------------------------------------------------------ decode (subtraction form)

DECODE = [k for k, w in PARITY_WORKLOADS.items() if w.mode == "decode"]
# The kept part cancels against the global state: besides the rounding of exp(q) and
# exp(k) (two roundings on the residual), the fp32 sums of the state and of the kept
# tokens differ by accumulation error relative to the whole cache's magnitude.
GLOBAL_REL = 2.0 ** -12


def test_decode_state_matches_oracle_and_adds_up():
    w = PARITY_WORKLOADS["d_bf16_blk64"]
    x, dev = inputs(w)
    st = spa.spa_rla_decode_state(dev["k"], dev["v"])
    torch.cuda.synchronize()
    o = oracle.rla_block_states(x["k"], x["v"], "bf16", w.T)[:, :, 0]
    m = oracle.rla_block_states(x["k"], abs_v(x)["v"], "bf16", w.T)[:, :, 0]
    within(st.cpu().numpy().astype(np.float64), o, m, "decode state", 1)
    st2 = spa.spa_rla_decode_state(dev["k"], dev["v"], 0, w.T - 5)
    spa.spa_rla_decode_state(dev["k"], dev["v"], w.T - 5, w.T, state=st2)
    torch.cuda.synchronize()
    within(st2.cpu().numpy().astype(np.float64), o, m, "decode state in two calls", 1)
    assert spa.spa_get_device_error() == 0


def decode_rla_check(w, x, dev, idx, cnt, what):
    st = spa.spa_rla_decode_state(dev["k"], dev["v"])
    out, orla = spa.spa_sparse_attn_decode_rla(dev["q"], dev["k"], dev["v"], st, w.block,
                                               torch.from_numpy(idx).cuda(),
                                               torch.from_numpy(cnt).cuda(), w.scale)
    torch.cuda.synchronize()
    g = orla.cpu().numpy().astype(np.float64)
    o, m = oracle.rla(x["q"], x["k"], x["v"], "bf16", w.block, idx, cnt)
    _, m_all = oracle.rla(x["q"], x["k"], x["v"], "bf16", w.block, idx, np.zeros_like(cnt))
    err = np.abs(g - o)
    bound = (2 + 0.2) * U_BF16 * m + GLOBAL_REL * m_all.max(axis=-1, keepdims=True)
    assert (err <= bound).all(), (what, float((err / bound).max()))
    # the exact branch is unchanged by the linear one
    ref = spa.spa_sparse_attn_decode(dev["q"], dev["k"], dev["v"], w.block,
                                     torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda(),
                                     w.scale)
    assert torch.equal(out, ref)
    print(f"\n{what}: worst err / bound = {float((err / bound).max()):.3e}, "
          f"residual share of magnitude {float(m.sum() / m_all.sum()):.3f}")
    assert spa.spa_get_device_error() == 0


@pytest.mark.parametrize("top_p", [None, 0.3])
@pytest.mark.parametrize("key", DECODE)
def test_decode_rla_on_oracle_lists(key, top_p):
    w = PARITY_WORKLOADS[key]
    x, dev = inputs(w)
    if top_p is not None:
        w = w.with_(top_p=top_p)
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    decode_rla_check(w, x, dev, sel["idx"], sel["count"], f"{w.name} p={w.top_p}")


def test_decode_rla_random_lists_and_edges():
    w = PARITY_WORKLOADS["d_bf16_blk16"]
    x, dev = inputs(w)
    rng = np.random.default_rng(5)
    idx = np.full((w.B, w.Hq, 1, w.nb), -1, np.int32)
    cnt = np.zeros((w.B, w.Hq, 1), np.int32)
    for b in range(w.B):
        for h in range(w.Hq):
            keep = [j for j in range(w.nb) if rng.random() < 0.5]
            if h == 1:
                keep = []                          # nothing kept: global linear attention
            if h == 2:
                keep = list(range(w.nb))           # everything kept: the branch is ~0
            idx[b, h, 0, :len(keep)] = keep
            cnt[b, h, 0] = len(keep)
    decode_rla_check(w, x, dev, idx, cnt, "random lists")
