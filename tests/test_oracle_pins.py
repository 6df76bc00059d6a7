"""Pins for the CPU oracle: closed forms, hand-worked examples, brute force,
invariants and special cases, none of which re-types the oracle's own formulas.

Each test names the passage it pins. CPU only.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _rand(shape, seed, scale=1.0):
    return (np.random.default_rng(seed).standard_normal(shape) * scale).astype(np.float32)


# ---------------------------------------------------------------- block statistics
# SPLA, section 2.1: first- and second-order block statistics (mean, diagonal variance).

def test_stats_match_numpy_mean_and_population_variance():
    k = _rand((2, 3, 37, 8), 1)            # 37 = 4 full blocks of 8 + a partial block of 5
    mean, var = oracle.block_stats(k, "f32", 8)
    assert mean.shape == (2, 3, 5, 8)
    for j in range(5):
        blk = k[:, :, 8 * j:8 * (j + 1), :].astype(np.float64)
        np.testing.assert_allclose(mean[:, :, j], blk.mean(axis=2), rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(var[:, :, j], blk.var(axis=2, ddof=0), rtol=1e-12, atol=1e-14)


def test_stats_two_key_closed_form():
    a, b = np.float32(1.5), np.float32(-0.25)
    k = np.array([[[[a, 0.0], [b, 2.0]]]], np.float32)
    mean, var = oracle.block_stats(k, "f32", 2)
    assert mean[0, 0, 0, 0] == (a + b) / 2 and mean[0, 0, 0, 1] == 1.0
    assert var[0, 0, 0, 0] == pytest.approx(((a - b) / 2) ** 2, rel=1e-15)
    assert var[0, 0, 0, 1] == pytest.approx(1.0, rel=1e-15)


def test_stats_invariant_under_permutation_within_block():
    k = _rand((1, 2, 64, 16), 2)
    perm = np.concatenate([np.random.default_rng(3).permutation(16) + 16 * j for j in range(4)])
    m0, v0 = oracle.block_stats(k, "f32", 16)
    m1, v1 = oracle.block_stats(k[:, :, perm], "f32", 16)
    np.testing.assert_allclose(m1, m0, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(v1, v0, rtol=1e-12, atol=1e-15)


def test_stats_read_bf16_bit_patterns():
    from workloads import bf16_bits, widen
    k32 = _rand((1, 1, 20, 8), 4)
    bits = bf16_bits(k32)
    m_b, v_b = oracle.block_stats(bits, "bf16", 8)
    m_f, v_f = oracle.block_stats(widen(bits, "bf16"), "f32", 8)
    assert np.array_equal(m_b, m_f) and np.array_equal(v_b, v_f)


# ---------------------------------------------------------------- Taylor score
# SPLA, section 2.1: the score approximates the block's integrated attention mass
# sum_u exp(s qbar . k_u) by a second-order expansion about the block mean.

def test_score_hand_worked_examples():
    g = _golden()["taylor_score"]
    for case in g["cases"]:
        k = np.array(case["k"], np.float32)[None, None]
        q = np.array(case["q"], np.float32)[None, None]
        mean, var = oracle.block_stats(k, "f32", case["block"])
        l = oracle.scores(q, "f32", mean, var, case["T"], case["block"], case["scale"])
        np.testing.assert_allclose(l[0, 0, -1, :len(case["expected_l"])], case["expected_l"],
                                   rtol=1e-15, atol=1e-15, err_msg=case["name"])


def _exact_log_mass(qbar, keys, s):
    z = s * keys.astype(np.float64) @ qbar
    m = z.max()
    return m + math.log(np.exp(z - m).sum())


def test_score_exact_when_block_keys_identical():
    # var = 0 => no approximation is left: l_j == log sum_u exp(s qbar.k_u) exactly.
    rng = np.random.default_rng(5)
    T, blk, d = 96, 16, 8
    keys = np.repeat(rng.standard_normal((T // blk, d)).astype(np.float32), blk, axis=0)
    q = rng.standard_normal((1, 1, 1, d)).astype(np.float32)
    mean, var = oracle.block_stats(keys[None, None], "f32", blk)
    assert np.all(var == 0)
    s = 0.3
    l = oracle.scores(q, "f32", mean, var, T, blk, s)[0, 0, 0]
    for j in range(T // blk):
        ref = _exact_log_mass(q[0, 0, 0].astype(np.float64), keys[j * blk:(j + 1) * blk], s)
        assert l[j] == pytest.approx(ref, rel=1e-13, abs=1e-13)


def test_score_exact_for_unit_blocks_and_pooled_prefill_query():
    rng = np.random.default_rng(6)
    T, d = 9, 4
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    q = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    mean, var = oracle.block_stats(k, "f32", 1)
    l = oracle.scores(q, "f32", mean, var, T, 1, 0.7)
    for i in range(T):
        for j in range(T):
            if j > i:
                assert l[0, 0, i, j] == -np.inf
            else:
                ref = 0.7 * float(q[0, 0, i].astype(np.float64) @ k[0, 0, j].astype(np.float64))
                assert l[0, 0, i, j] == pytest.approx(ref, rel=1e-13, abs=1e-14)


def _diag_cov_block(d, rng):
    """3d keys whose deviations from the mean lie on single axes: the sample
    covariance is exactly diagonal and the third moment is non-zero."""
    mu = rng.standard_normal(d)
    a = 0.5 + rng.random(d)
    rows = []
    for c in range(d):
        e = np.zeros(d)
        e[c] = a[c]
        rows += [mu + 2 * e, mu - e, mu - e]
    return np.array(rows, np.float64).astype(np.float32)


def test_score_error_is_third_order_in_query_norm():
    # With a diagonal covariance, exact log mass - l = O(|q|^3) (second-order
    # expansion). A dropped 1/2, a dropped s^2, a wrong sign or a std in place of a
    # variance leaves an O(|q|^2) error; a wrong mean term leaves O(|q|).
    rng = np.random.default_rng(7)
    d = 6
    keys = _diag_cov_block(d, rng)
    blk = keys.shape[0]
    mean, var = oracle.block_stats(keys[None, None], "f32", blk)
    direction = rng.standard_normal(d)
    s = 1 / math.sqrt(d)
    errs = []
    for eps in [0.2, 0.1, 0.05, 0.025]:
        qv = (eps * direction).astype(np.float32)
        l = oracle.scores(qv[None, None, None], "f32", mean, var, blk, blk, s)[0, 0, 0, 0]
        errs.append(abs(_exact_log_mass(qv.astype(np.float64), keys, s) - l))
    ratios = [errs[n] / errs[n + 1] for n in range(3)]
    assert all(6.5 < r < 9.5 for r in ratios), (errs, ratios)


def test_score_gqa_head_reads_its_group():
    rng = np.random.default_rng(8)
    B, Hq, Hkv, T, d, blk = 2, 4, 2, 40, 8, 8
    q = rng.standard_normal((B, Hq, T, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    mean, var = oracle.block_stats(k, "f32", blk)
    l = oracle.scores(q, "f32", mean, var, T, blk, 0.35)
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            one = oracle.scores(q[b:b + 1, h:h + 1], "f32", mean[b:b + 1, g:g + 1],
                                var[b:b + 1, g:g + 1], T, blk, 0.35)
            np.testing.assert_array_equal(l[b, h], one[0, 0])


# ---------------------------------------------------------------- dual top-p cut
# SpotAttention, section 3: reserved sink/recency blocks, nucleus over the residual,
# K_min floor.

def test_top_p_hand_worked_examples():
    g = _golden()["top_p"]
    l = np.array(g["scores"], np.float64)[None, None, None]
    T = 6 * 4
    for case in g["cases"]:
        idx, cnt = oracle.select_from_scores(l, 1, T, 4, case["top_p"], 1, 1, case["k_min"])
        got = list(idx[0, 0, 0, :cnt[0, 0, 0]])
        assert got == case["expected"], (case, got)
        assert np.all(idx[0, 0, 0, cnt[0, 0, 0]:] == -1)


def _brute_force_keep(scores32, p, k_min):
    """Smallest subset of the residual whose normalised mass reaches p (the
    heaviest such subset), then padded to the K_min heaviest."""
    n = len(scores32)
    w = np.exp(scores32.astype(np.float64) - scores32.max())
    w /= w.sum()
    order = sorted(range(n), key=lambda j: (-scores32[j], j))
    best = None
    if p >= 1:
        best = set(range(n))
    else:
        for c in range(1, n + 1):
            cands = [S for S in itertools.combinations(range(n), c) if w[list(S)].sum() >= p]
            if cands:
                top = max(w[list(S)].sum() for S in cands)
                best = set(min(S for S in cands if w[list(S)].sum() == top))
                break
    floor = min(k_min, n)
    if len(best) < floor:
        best = set(order[:floor])
    return best


@pytest.mark.parametrize("seed", range(40))
def test_top_p_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    jmax = int(rng.integers(0, 14))
    n_sink, n_local = int(rng.integers(0, 3)), int(rng.integers(0, 3))
    k_min = int(rng.choice([0, 0, 1, 3]))
    p = float(rng.choice([rng.random(), 1.0, rng.random() * 0.3]))
    p = max(p, 1e-6)
    blk = 4
    T = (jmax + 1) * blk
    l = rng.standard_normal(jmax + 1) * 2.0
    idx, cnt = oracle.select_from_scores(l[None, None, None], 1, T, blk, p, n_sink, n_local, k_min)
    got = set(idx[0, 0, 0, :cnt[0, 0, 0]].tolist())
    rsv = {j for j in range(jmax + 1) if j < n_sink or j > jmax - n_local}
    resid = [j for j in range(jmax + 1) if j not in rsv]
    exp = set(rsv)
    if resid:
        s32 = l[resid].astype(np.float32)
        # skip cases whose decision sits within rounding of p
        w = np.exp(s32.astype(np.float64) - s32.max())
        w /= w.sum()
        cum = np.cumsum(np.sort(w)[::-1])
        if p < 1 and np.any(np.abs(cum - p) < 1e-9):
            pytest.skip("boundary case")
        exp |= {resid[j] for j in _brute_force_keep(s32, p, k_min)}
    assert got == exp
    assert list(idx[0, 0, 0, :cnt[0, 0, 0]]) == sorted(exp)


def test_top_p_tiny_p_keeps_top_one():
    l = np.array([0.0, 0.5, 3.0, -1.0, 2.9, 0.0])[None, None, None]
    idx, cnt = oracle.select_from_scores(l, 1, 6, 1, 1e-9, 1, 1)
    assert list(idx[0, 0, 0, :cnt[0, 0, 0]]) == [0, 2, 5]


def test_top_p_equal_scores_prefer_smaller_index():
    l = np.zeros((1, 1, 1, 6))
    idx, cnt = oracle.select_from_scores(l, 1, 6, 1, 0.5, 1, 1)   # residual 1..4, 1/4 each
    assert list(idx[0, 0, 0, :cnt[0, 0, 0]]) == [0, 1, 2, 5]


def test_top_p_prefill_reserved_blocks_and_causal_limit():
    rng = np.random.default_rng(9)
    nq = 7
    l = rng.standard_normal((1, 2, nq, nq))
    l[..., np.triu_indices(nq, 1)[0], np.triu_indices(nq, 1)[1]] = -np.inf
    idx, cnt = oracle.select_from_scores(l, nq * 8, nq * 8, 8, 0.3, 1, 1)
    for h in range(2):
        for i in range(nq):
            lst = idx[0, h, i, :cnt[0, h, i]].tolist()
            assert lst == sorted(set(lst))
            assert 0 in lst and i in lst and max(lst) == i
    assert cnt[0, 0, 0] == 1 and cnt[0, 0, 1] == 2


# ---------------------------------------------------------------- attention
# S2O, section 3: exact softmax attention over the selected blocks.

def test_attention_hand_worked_example():
    g = _golden()["attention"]
    T, d, blk = g["T"], g["d"], g["block"]
    q = np.array(g["q"], np.float32).reshape(1, 1, T, d)
    k = np.array(g["k"], np.float32).reshape(1, 1, T, d)
    v = np.array(g["v"], np.float32).reshape(1, 1, T, d)
    idx, cnt = oracle.full_lists(1, 1, T, T, blk)
    out, lse = oracle.attention(q, k, v, "f32", blk, idx, cnt, g["scale"])
    np.testing.assert_allclose(out[0, 0, :, 0], g["expected_prefill_out"], rtol=1e-14)
    np.testing.assert_allclose(lse[0, 0], g["expected_prefill_lse"], rtol=1e-14, atol=1e-15)


def _random_lists(B, Hq, T, blk, seed):
    rng = np.random.default_rng(seed)
    nb = -(-T // blk)
    idx = np.full((B, Hq, nb, nb), -1, np.int32)
    cnt = np.zeros((B, Hq, nb), np.int32)
    for b in range(B):
        for h in range(Hq):
            for i in range(nb):
                keep = sorted({0, i} | {j for j in range(i + 1) if rng.random() < 0.5})
                idx[b, h, i, :len(keep)] = keep
                cnt[b, h, i] = len(keep)
    return idx, cnt


def test_attention_constant_keys_average_allowed_values():
    # Equal logits => the output is the plain mean of the allowed values
    # (u <= t and block(u) kept): pins the mask and the normalisation.
    rng = np.random.default_rng(10)
    B, Hq, Hkv, T, d, blk = 1, 2, 1, 45, 4, 8
    q = rng.standard_normal((B, Hq, T, d)).astype(np.float32)
    k = np.tile(rng.standard_normal(d).astype(np.float32), (B, Hkv, T, 1))
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    idx, cnt = _random_lists(B, Hq, T, blk, 11)
    out, _ = oracle.attention(q, k, v, "f32", blk, idx, cnt, 0.5)
    for h in range(Hq):
        for t in range(T):
            kept = set(idx[0, h, t // blk, :cnt[0, h, t // blk]].tolist())
            allowed = [u for u in range(t + 1) if u // blk in kept]
            np.testing.assert_allclose(out[0, h, t], v[0, 0, allowed].astype(np.float64).mean(0),
                                       rtol=1e-12, atol=1e-13)


def test_attention_constant_values_and_dominant_key():
    rng = np.random.default_rng(12)
    T, d, blk = 30, 4, 8
    q = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    c = rng.standard_normal(d).astype(np.float32)
    v = np.tile(c, (1, 1, T, 1))
    idx, cnt = _random_lists(1, 1, T, blk, 13)
    out, _ = oracle.attention(q, k, v, "f32", blk, idx, cnt, 0.4)
    np.testing.assert_allclose(out[0, 0], np.tile(c.astype(np.float64), (T, 1)), rtol=1e-12)
    # one key with a huge logit for every query that can see it
    k2 = k.copy()
    k2[0, 0, 3] = 0
    q2 = q.copy()
    q2[0, 0, :, 0] = 1
    k2[0, 0, 3, 0] = 200.0
    v2 = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    full_i, full_c = oracle.full_lists(1, 1, T, T, blk)
    out2, _ = oracle.attention(q2, k2, v2, "f32", blk, full_i, full_c, 1.0)
    np.testing.assert_allclose(out2[0, 0, 3:], np.tile(v2[0, 0, 3].astype(np.float64), (T - 3, 1)),
                               rtol=1e-12, atol=1e-12)


def _dense_causal_numpy(q, k, v, s):
    B, Hq, L, d = q.shape
    G = Hq // k.shape[1]
    out = np.empty(q.shape, np.float64)
    mask = np.tril(np.ones((L, L), bool))
    for b in range(B):
        for h in range(Hq):
            z = s * q[b, h].astype(np.float64) @ k[b, h // G].astype(np.float64).T
            z = np.where(mask, z, -np.inf)
            z -= z.max(axis=1, keepdims=True)
            p = np.exp(z)
            p /= p.sum(axis=1, keepdims=True)
            out[b, h] = p @ v[b, h // G].astype(np.float64)
    return out


@pytest.mark.parametrize("T,blk", [(64, 16), (70, 16), (33, 64)])
def test_top_p_one_equals_dense_causal_attention(T, blk):
    rng = np.random.default_rng(14 + T)
    B, Hq, Hkv, d = 2, 4, 2, 8
    q = rng.standard_normal((B, Hq, T, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    s = 1 / math.sqrt(d)
    sel = oracle.select(q, k, "f32", blk, s, 1.0)
    nq = -(-T // blk)
    for i in range(nq):
        assert np.all(sel["count"][:, :, i] == i + 1)
    out, _ = oracle.attention(q, k, v, "f32", blk, sel["idx"], sel["count"], s)
    np.testing.assert_allclose(out, _dense_causal_numpy(q, k, v, s), rtol=1e-11, atol=1e-12)


def test_single_block_sequence_is_dense_causal_at_any_p():
    rng = np.random.default_rng(15)
    for T in (16, 11):
        q = rng.standard_normal((1, 2, T, 8)).astype(np.float32)
        k = rng.standard_normal((1, 1, T, 8)).astype(np.float32)
        v = rng.standard_normal((1, 1, T, 8)).astype(np.float32)
        sel = oracle.select(q, k, "f32", 16, 0.3, 0.1)
        out, _ = oracle.attention(q, k, v, "f32", 16, sel["idx"], sel["count"], 0.3)
        np.testing.assert_allclose(out, _dense_causal_numpy(q, k, v, 0.3), rtol=1e-11, atol=1e-12)


def test_kv_permutation_within_earlier_blocks_changes_nothing():
    # Sparsere Blok-Sparse Attention via Tokenpermutatie, section 1: attention is
    # invariant under a joint permutation of (k, v) pairs; within a block that lies
    # wholly before the query block the stats (up to rounding), the selection and
    # the output of the last query block are unchanged.
    rng = np.random.default_rng(16)
    B, Hq, Hkv, T, d, blk = 1, 4, 2, 96, 8, 16
    q = rng.standard_normal((B, Hq, T, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    perm = np.arange(T)
    for j in range(T // blk - 1):
        perm[j * blk:(j + 1) * blk] = j * blk + rng.permutation(blk)
    s = 1 / math.sqrt(d)
    a = oracle.select(q, k, "f32", blk, s, 0.7)
    b = oracle.select(q, k[:, :, perm], "f32", blk, s, 0.7)
    np.testing.assert_allclose(b["mean"], a["mean"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(b["var"], a["var"], rtol=1e-12, atol=1e-15)
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["count"], b["count"])
    rows = np.array([(h * T + t) for h in range(Hq) for t in range(T - blk, T)])
    oa, _ = oracle.attention(q, k, v, "f32", blk, a["idx"], a["count"], s, rows=rows)
    ob, _ = oracle.attention(q, k[:, :, perm], v[:, :, perm], "f32", blk, b["idx"], b["count"], s,
                             rows=rows)
    np.testing.assert_allclose(ob, oa, rtol=1e-12, atol=1e-13)


def test_segmented_permutation_keeps_later_segments_at_p_one():
    # Same page, section 2: permuting within a segment of size S keeps every query
    # of a later segment unchanged (all of the segment lies in its causal past).
    rng = np.random.default_rng(17)
    T, d, blk, S = 64, 8, 8, 16
    q = rng.standard_normal((1, 2, T, d)).astype(np.float32)
    k = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    v = rng.standard_normal((1, 1, T, d)).astype(np.float32)
    perm = np.concatenate([seg * S + rng.permutation(S) for seg in range(T // S)])
    fi, fc = oracle.full_lists(1, 2, T, T, blk)
    oa, _ = oracle.attention(q, k, v, "f32", blk, fi, fc, 0.3)
    for seg in range(T // S):
        p = np.arange(T)
        p[seg * S:(seg + 1) * S] = perm[seg * S:(seg + 1) * S]
        ob, _ = oracle.attention(q, k[:, :, p], v[:, :, p], "f32", blk, fi, fc, 0.3)
        later = slice((seg + 1) * S, T)
        np.testing.assert_allclose(ob[:, :, later], oa[:, :, later], rtol=1e-12, atol=1e-13)
        if seg < T // S - 1:
            assert not np.allclose(ob[:, :, seg * S:(seg + 1) * S], oa[:, :, seg * S:(seg + 1) * S])


def test_decode_equals_prefill_last_row():
    rng = np.random.default_rng(18)
    B, Hq, Hkv, T, d, blk = 2, 4, 2, 77, 8, 16
    q = rng.standard_normal((B, Hq, T, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    s = 0.33
    qd = q[:, :, T - 1:T].copy()
    dec = oracle.select(qd, k, "f32", blk, s, 0.6)
    od, lse_d = oracle.attention(qd, k, v, "f32", blk, dec["idx"], dec["count"], s)
    # prefill lists: every query block keeps everything, except the last one, which
    # takes the decode list
    nq = -(-T // blk)
    pi, pc = oracle.full_lists(B, Hq, T, T, blk)
    pi[:, :, nq - 1] = dec["idx"][:, :, 0]
    pc[:, :, nq - 1] = dec["count"][:, :, 0]
    op, lse_p = oracle.attention(q, k, v, "f32", blk, pi, pc, s)
    np.testing.assert_allclose(od[:, :, 0], op[:, :, T - 1], rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse_d[:, :, 0], lse_p[:, :, T - 1], rtol=1e-13)
    # decode at p = 1 is dense attention of one query over the whole cache
    full = oracle.select(qd, k, "f32", blk, s, 1.0)
    of, _ = oracle.attention(qd, k, v, "f32", blk, full["idx"], full["count"], s)
    ref = _dense_causal_numpy(q, k, v, s)[:, :, T - 1]
    np.testing.assert_allclose(of[:, :, 0], ref, rtol=1e-11, atol=1e-12)


def test_attention_rows_subset_matches_full():
    rng = np.random.default_rng(19)
    B, Hq, Hkv, T, d, blk = 1, 4, 2, 50, 8, 8
    q = rng.standard_normal((B, Hq, T, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    idx, cnt = _random_lists(B, Hq, T, blk, 20)
    full, lse = oracle.attention(q, k, v, "f32", blk, idx, cnt, 0.3)
    rows = np.array([0, 5, 49, 50, 123, 199])
    part, lse_p = oracle.attention(q, k, v, "f32", blk, idx, cnt, 0.3, rows=rows)
    np.testing.assert_array_equal(part, full.reshape(-1, d)[rows])
    np.testing.assert_array_equal(lse_p, lse.reshape(-1)[rows])


def test_attention_gqa_head_reads_its_group():
    rng = np.random.default_rng(21)
    B, Hq, Hkv, T, d, blk = 1, 6, 3, 40, 4, 8
    q = rng.standard_normal((B, Hq, T, d)).astype(np.float32)
    k = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    v = rng.standard_normal((B, Hkv, T, d)).astype(np.float32)
    idx, cnt = _random_lists(B, Hq, T, blk, 22)
    out, _ = oracle.attention(q, k, v, "f32", blk, idx, cnt, 0.5)
    for h in range(Hq):
        g = h // 2
        one, _ = oracle.attention(q[:, h:h + 1], k[:, g:g + 1], v[:, g:g + 1], "f32", blk,
                                  idx[:, h:h + 1], cnt[:, h:h + 1], 0.5)
        np.testing.assert_array_equal(out[:, h], one[:, 0])


def test_oracle_rejects_bad_lists():
    q = np.zeros((1, 1, 8, 4), np.float32)
    idx = np.array([[[[0, 5]]]], np.int32)            # block 5 does not exist
    cnt = np.array([[[2]]], np.int32)
    with pytest.raises(RuntimeError):
        oracle.attention(q, q, q, "f32", 8, idx, cnt, 1.0)


# ---------------------------------------------------------------- residual linear attention
# SPLA, sections 2.2-2.3: the unkept blocks enter a linear-attention branch with the
# feature map phi = exp; its output is the global linear attention minus the linear
# attention over the kept blocks.

def _rla_golden_inputs(g):
    q = np.array(g["q"], np.float32)[None, None]
    k = np.array(g["k"], np.float32)[None, None]
    v = np.array(g["v"], np.float32)[None, None]
    return q, k, v


def test_rla_hand_worked_examples():
    g = _golden()["rla"]
    q, k, v = _rla_golden_inputs(g)
    for tag in ("A", "B"):
        lists = g["lists_" + tag]
        idx = np.array(lists["idx"], np.int32)[None, None]
        cnt = np.array(lists["count"], np.int32)[None, None]
        out, mag = oracle.rla(q, k, v, "f32", g["block"], idx, cnt)
        np.testing.assert_allclose(out[0, 0], np.array(g["expected_" + tag]), rtol=1e-14, atol=1e-14)
        if tag == "B":
            np.testing.assert_allclose(mag[0, 0, 3], g["expected_B_mag_row3"], rtol=1e-14)
    dl = g["decode_list"]
    out, _ = oracle.rla(q[:, :, 3:4], k, v, "f32", g["block"],
                        np.array(dl["idx"], np.int32).reshape(1, 1, 1, 2),
                        np.array([dl["count"]], np.int32).reshape(1, 1, 1))
    np.testing.assert_allclose(out[0, 0, 0], g["expected_decode"], rtol=1e-14)


def test_rla_is_zero_when_every_causal_block_is_kept():
    q, k, v = _rand((1, 4, 70, 8), 41, 0.5), _rand((1, 2, 70, 8), 42, 0.5), _rand((1, 2, 70, 8), 43)
    idx, cnt = oracle.full_lists(1, 4, 70, 70, 16)
    out, mag = oracle.rla(q, k, v, "f32", 16, idx, cnt)
    assert np.all(out == 0.0) and np.all(mag == 0.0)


def _residual_token_mask(idx, cnt, Lq, T, block, b, h, t):
    i = t // block
    kept = set(int(j) for j in idx[b, h, i, :cnt[b, h, i]])
    pos = T - Lq + t
    return np.array([(u <= pos) and (u // block not in kept) for u in range(T)])


def test_rla_unit_features_sum_residual_values():
    # q = k = 0: phi = 1, every weight is d, so the output is d times the plain sum of
    # the residual tokens' values.
    B, Hq, Hkv, T, d, blk = 1, 2, 1, 40, 4, 8
    q = np.zeros((B, Hq, T, d), np.float32)
    k = np.zeros((B, Hkv, T, d), np.float32)
    v = _rand((B, Hkv, T, d), 44)
    idx, cnt = _random_lists(B, Hq, T, blk, 45)
    out, _ = oracle.rla(q, k, v, "f32", blk, idx, cnt)
    for h in range(Hq):
        for t in range(T):
            m = _residual_token_mask(idx, cnt, T, T, blk, 0, h, t)
            np.testing.assert_allclose(out[0, h, t], d * v[0, 0][m].astype(np.float64).sum(axis=0),
                                       rtol=1e-13, atol=1e-13)


def test_rla_global_minus_kept_equals_residual():
    # The subtraction form: linear attention over every causal token (global),
    # minus that over the kept blocks, is the residual branch. Global and kept parts
    # are evaluated here as masked matrix products.
    B, Hq, Hkv, T, d, blk = 1, 2, 2, 48, 6, 8
    q, k, v = _rand((B, Hq, T, d), 46, 0.4), _rand((B, Hkv, T, d), 47, 0.4), _rand((B, Hkv, T, d), 48)
    # lists that may leave out the sink and the query's own (diagonal) block
    rng = np.random.default_rng(49)
    nb = T // blk
    idx = np.full((B, Hq, nb, nb), -1, np.int32)
    cnt = np.zeros((B, Hq, nb), np.int32)
    for h in range(Hq):
        for i in range(nb):
            keep = [j for j in range(i + 1) if rng.random() < 0.5]
            idx[0, h, i, :len(keep)] = keep
            cnt[0, h, i] = len(keep)
    assert any(cnt[0, h, i] == 0 or idx[0, h, i, cnt[0, h, i] - 1] != i
               for h in range(Hq) for i in range(nb))
    out, _ = oracle.rla(q, k, v, "f32", blk, idx, cnt)
    for h in range(Hq):
        A = np.exp(q[0, h].astype(np.float64)) @ np.exp(k[0, h].astype(np.float64)).T
        causal = np.tril(np.ones((T, T)))
        kept = np.zeros((T, T))
        for t in range(T):
            i = t // blk
            for j in idx[0, h, i, :cnt[0, h, i]]:
                kept[t, j * blk:(j + 1) * blk] = 1
        kept *= causal
        o_global = (A * causal) @ v[0, h].astype(np.float64)
        o_kept = (A * kept) @ v[0, h].astype(np.float64)
        np.testing.assert_allclose(out[0, h], o_global - o_kept, rtol=1e-10, atol=1e-10)


def test_rla_block_states_contract_to_residual_output():
    # The chunked form: W_j = (phi(K_j)^T V_j)^T per block; a row whose own block is
    # kept gets phi(q_t) contracted with the sum of W_j over its residual blocks.
    B, Hq, Hkv, T, d, blk = 1, 4, 2, 64, 8, 16
    q, k, v = _rand((B, Hq, T, d), 50, 0.4), _rand((B, Hkv, T, d), 51, 0.4), _rand((B, Hkv, T, d), 52)
    W = oracle.rla_block_states(k, v, "f32", blk)
    nb = T // blk
    for g in range(Hkv):
        for j in range(nb):
            Kj = np.exp(k[0, g, j * blk:(j + 1) * blk].astype(np.float64))
            Vj = v[0, g, j * blk:(j + 1) * blk].astype(np.float64)
            np.testing.assert_allclose(W[0, g, j], (Kj.T @ Vj).T, rtol=1e-12)
    idx, cnt = oracle.full_lists(B, Hq, T, T, blk)
    rng = np.random.default_rng(53)
    for h in range(Hq):
        for i in range(nb):
            keep = [j for j in range(i) if rng.random() < 0.5] + [i]
            idx[0, h, i, :] = -1
            idx[0, h, i, :len(keep)] = keep
            cnt[0, h, i] = len(keep)
    out, _ = oracle.rla(q, k, v, "f32", blk, idx, cnt)
    for h in range(Hq):
        g = h // (Hq // Hkv)
        for i in range(nb):
            res = [j for j in range(i) if j not in set(idx[0, h, i, :cnt[0, h, i]])]
            S = sum((W[0, g, j] for j in res), np.zeros((d, d)))
            rows = np.exp(q[0, h, i * blk:(i + 1) * blk].astype(np.float64))
            np.testing.assert_allclose(out[0, h, i * blk:(i + 1) * blk], rows @ S.T, rtol=1e-11,
                                       atol=1e-11)


def test_rla_query_shift_scales_output():
    # phi(q + c) = e^c phi(q) component-wise, so a uniform shift of the query scales
    # the branch output by e^c (a dot-product feature map would not do this).
    B, Hq, Hkv, T, d, blk = 1, 1, 1, 32, 4, 8
    q, k, v = _rand((B, Hq, T, d), 54, 0.5), _rand((B, Hkv, T, d), 55, 0.5), _rand((B, Hkv, T, d), 56)
    idx, cnt = _random_lists(B, Hq, T, blk, 57)
    o0, _ = oracle.rla(q, k, v, "f32", blk, idx, cnt)
    o1, _ = oracle.rla(q + np.float32(0.75), k, v, "f32", blk, idx, cnt)
    np.testing.assert_allclose(o1, o0 * math.exp(0.75), rtol=1e-6)


def test_rla_ignores_future_tokens_and_kept_blocks():
    B, Hq, Hkv, T, d, blk = 1, 2, 1, 48, 4, 8
    q, k, v = _rand((B, Hq, T, d), 58, 0.5), _rand((B, Hkv, T, d), 59, 0.5), _rand((B, Hkv, T, d), 60)
    idx, cnt = _random_lists(B, Hq, T, blk, 61)
    out, _ = oracle.rla(q, k, v, "f32", blk, idx, cnt)
    t = 27                               # row in query block 3
    k2, v2 = k.copy(), v.copy()
    k2[:, :, t + 1:] += 3.0              # future tokens
    v2[:, :, t + 1:] -= 5.0
    for h in range(Hq):
        for j in idx[0, h, 3, :cnt[0, h, 3]]:
            if h == 0:                   # blocks head 0 keeps for this query block
                k2[:, :, j * blk:min((j + 1) * blk, t + 1)] *= 2.0
    out2, _ = oracle.rla(q, k2, v2, "f32", blk, idx, cnt)
    np.testing.assert_allclose(out2[0, 0, t], out[0, 0, t], rtol=1e-13, atol=1e-13)


def test_rla_decode_equals_prefill_last_row():
    B, Hq, Hkv, T, d, blk = 2, 4, 2, 45, 4, 8
    q, k, v = _rand((B, Hq, T, d), 62, 0.5), _rand((B, Hkv, T, d), 63, 0.5), _rand((B, Hkv, T, d), 64)
    idx, cnt = _random_lists(B, Hq, T, blk, 65)
    out, _ = oracle.rla(q, k, v, "f32", blk, idx, cnt)
    i = (T - 1) // blk
    od, _ = oracle.rla(q[:, :, T - 1:T], k, v, "f32", blk, idx[:, :, i:i + 1], cnt[:, :, i:i + 1])
    np.testing.assert_allclose(od[:, :, 0], out[:, :, T - 1], rtol=1e-13, atol=1e-13)


def test_rla_gqa_head_reads_its_group():
    B, Hq, Hkv, T, d, blk = 1, 4, 2, 32, 4, 8
    q = np.repeat(_rand((B, 1, T, d), 66, 0.5), Hq, axis=1)
    k, v = _rand((B, Hkv, T, d), 67, 0.5), _rand((B, Hkv, T, d), 68)
    idx, cnt = oracle.full_lists(B, Hq, T, T, blk)
    idx[:, :, 3, :] = -1
    idx[:, :, 3, 0] = 3
    cnt[:, :, 3] = 1
    out, _ = oracle.rla(q, k, v, "f32", blk, idx, cnt)
    np.testing.assert_array_equal(out[0, 0], out[0, 1])
    np.testing.assert_array_equal(out[0, 2], out[0, 3])
    assert np.abs(out[0, 0, 31] - out[0, 2, 31]).max() > 1e-3
    ref, _ = oracle.rla(q[:, 2:3], k[:, 1:2], v[:, 1:2], "f32", blk, idx[:, 2:3], cnt[:, 2:3])
    np.testing.assert_array_equal(out[0, 2], ref[0, 0])


# ---------------------------------------------------------------- quantised statistics
# SpotAttention, section 4: the selector's cache in INT4 microscale (format as read:
# power-of-two scale per 32 features, round half to even).

def test_quantized_stats_hand_worked_group():
    g = _golden()["quantized_stats"]
    mean = np.array(g["mean_group"], np.float64).reshape(1, 1, 1, 32)
    var = np.array(g["var_group"], np.float64).reshape(1, 1, 1, 32)
    qs = oracle.quantize_stats(mean, var)
    assert int(qs["km"][0, 0, 0, 0]) == g["expected_km"]
    assert int(qs["kv"][0, 0, 0, 0]) == g["expected_kv"]
    assert qs["cm"].reshape(-1).tolist() == g["expected_cm"]
    assert qs["cv"].reshape(-1).tolist() == g["expected_cv"]


def _quant_inputs(seed):
    rng = np.random.default_rng(seed)
    mean = rng.standard_normal((2, 2, 5, 64)) * np.exp(rng.uniform(-6, 6, (2, 2, 5, 2)))[..., None].repeat(32, -1).reshape(2, 2, 5, 64)
    var = rng.exponential(1.0, (2, 2, 5, 64)) * 10.0 ** rng.integers(-3, 3, (2, 2, 5, 1))
    mean[0, 0, 1, :32] = 0.0                   # an all-zero group
    var[1, 1, 2, 32:] = 0.0
    return mean, var


def test_quantized_stats_error_and_scale_bounds():
    mean, var = _quant_inputs(70)
    qs = oracle.quantize_stats(mean, var)
    dm, dv = oracle.dequantize_stats(qs)
    m32, v32 = mean.astype(np.float32).astype(np.float64), var.astype(np.float32).astype(np.float64)
    step_m = np.ldexp(1.0, qs["km"].astype(np.int64)).repeat(32, axis=-1)
    step_v = np.ldexp(1.0, qs["kv"].astype(np.int64)).repeat(32, axis=-1)
    assert np.all(np.abs(dm - m32) <= step_m / 2) and np.all(np.abs(dv - v32) <= step_v / 2)
    assert qs["cm"].min() >= -7 and qs["cm"].max() <= 7 and qs["cv"].max() <= 15
    gm = np.abs(m32).reshape(2, 2, 5, 2, 32).max(-1)
    gv = v32.reshape(2, 2, 5, 2, 32).max(-1)
    km, kv = qs["km"].astype(np.int64), qs["kv"].astype(np.int64)
    nz = gm > 0
    # the scale is the smallest power of two that covers the group maximum
    assert np.all(gm[nz] <= 7 * np.ldexp(1.0, km[nz])) and np.all(gm[nz] > 7 * np.ldexp(1.0, km[nz] - 1))
    nzv = gv > 0
    assert np.all(gv[nzv] <= 15 * np.ldexp(1.0, kv[nzv])) and np.all(gv[nzv] > 15 * np.ldexp(1.0, kv[nzv] - 1))
    assert np.all(dm[0, 0, 1, :32] == 0) and np.all(dv[1, 1, 2, 32:] == 0)


def test_quantized_stats_power_of_two_scaling_shifts_only_the_exponent():
    mean, var = _quant_inputs(71)
    q0 = oracle.quantize_stats(mean, var)
    q1 = oracle.quantize_stats(mean * 2.0 ** 5, var * 2.0 ** -3)
    assert np.array_equal(q0["cm"], q1["cm"]) and np.array_equal(q0["cv"], q1["cv"])
    nzm = np.abs(mean).reshape(2, 2, 5, 2, 32).max(-1) > 0
    nzv = var.reshape(2, 2, 5, 2, 32).max(-1) > 0
    assert np.all(q1["km"][nzm].astype(int) == q0["km"][nzm].astype(int) + 5)
    assert np.all(q1["kv"][nzv].astype(int) == q0["kv"][nzv].astype(int) - 3)


def test_quantized_stats_on_the_grid_round_trip_exactly():
    rng = np.random.default_rng(72)
    codes_m = rng.integers(-7, 8, (1, 2, 3, 64))
    codes_m[..., 0] = 7                         # every group reaches the top code
    codes_m[..., 32] = -7
    codes_v = rng.integers(0, 16, (1, 2, 3, 64))
    codes_v[..., 0] = 15
    codes_v[..., 32] = 15
    mean = codes_m * 2.0 ** -4
    var = codes_v * 2.0 ** 3
    qs = oracle.quantize_stats(mean, var)
    dm, dv = oracle.dequantize_stats(qs)
    assert np.array_equal(dm, mean) and np.array_equal(dv, var)
    assert np.all(qs["km"] == -4) and np.all(qs["kv"] == 3)


def test_quantized_selection_equals_plain_selection_on_grid_statistics():
    # keys constant within a block and on a coarse grid: mean exactly on the grid,
    # variance 0, so quantisation changes nothing and neither does the selection
    rng = np.random.default_rng(73)
    B, Hq, Hkv, T, d, blk = 1, 4, 2, 256, 64, 32
    vals = rng.integers(-7, 8, (B, Hkv, T // blk, d)).astype(np.float32) * np.float32(0.125)
    vals[..., 0] = 7 * 0.125
    vals[..., 32] = -7 * 0.125
    k = np.repeat(vals, blk, axis=2)
    q = _rand((B, Hq, T, d), 74)
    a = oracle.select(q, k, "f32", blk, 0.125, 0.6)
    b = oracle.select_quantized(q, k, "f32", blk, 0.125, 0.6)
    assert np.array_equal(a["count"], b["count"]) and np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["scores"], b["scores"])


# FP4 records: the same section's other format, read as the OCP microscaling
# element E2M1 with the records' power-of-two scale per 32 features.

E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]   # the E2M1 magnitudes, codes 0..7


def test_fp4_stats_hand_worked_group():
    g = _golden()["quantized_stats_fp4"]
    mean = np.array(g["mean_group"], np.float64).reshape(1, 1, 1, 32)
    var = np.array(g["var_group"], np.float64).reshape(1, 1, 1, 32)
    qs = oracle.quantize_stats(mean, var, "fp4")
    assert int(qs["km"][0, 0, 0, 0]) == g["expected_km"]
    assert int(qs["kv"][0, 0, 0, 0]) == g["expected_kv"]
    assert qs["cm"].reshape(-1).tolist() == g["expected_cm"]
    assert qs["cv"].reshape(-1).tolist() == g["expected_cv"]


def test_fp4_codes_decode_to_the_e2m1_values():
    # code s e1 e0 m: (-1)^s 2^(e - 1) (1 + m / 2) for e > 0, (-1)^s m / 2 for e = 0
    codes = np.tile(np.arange(16, dtype=np.uint8), 2).reshape(1, 1, 1, 32)
    k = np.zeros((1, 1, 1, 1), np.int8)
    dm, dv = oracle.dequantize_stats({"cm": codes, "cv": codes, "km": k, "kv": k + 3, "fmt": "fp4"})
    want = [sgn * v for sgn in (1.0, -1.0) for v in E2M1_TABLE]
    assert dm.reshape(-1)[:16].tolist() == want
    assert dv.reshape(-1)[:16].tolist() == [8.0 * x for x in want]
    assert np.signbit(dm.reshape(-1)[8])                      # code 8 is -0


def _fp4_inputs(seed):
    rng = np.random.default_rng(seed)
    mean = rng.standard_normal((2, 2, 5, 64)) * np.exp(rng.uniform(-6, 6, (2, 2, 5, 2))).repeat(32, -1)
    var = rng.exponential(1.0, (2, 2, 5, 64)) * 10.0 ** rng.integers(-3, 3, (2, 2, 5, 1))
    mean[0, 0, 1, :32] = 0.0                   # an all-zero group
    var[1, 1, 2, 32:] = 0.0
    return mean, var


def test_fp4_error_and_scale_bounds():
    mean, var = _fp4_inputs(80)
    qs = oracle.quantize_stats(mean, var, "fp4")
    dm, dv = oracle.dequantize_stats(qs)
    for x, d, k in ((mean, dm, qs["km"]), (var, dv, qs["kv"])):
        x32 = x.astype(np.float32).astype(np.float64)
        sc = np.ldexp(1.0, k.astype(np.int64)).repeat(32, axis=-1)
        a = np.abs(x32) / sc                    # in [0, 6]
        half_gap = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))
        assert np.all(np.abs(d - x32) <= half_gap * sc)
        assert np.all(np.sign(d) * np.sign(x32) >= 0)
        gmax = np.abs(x32).reshape(2, 2, 5, 2, 32).max(-1)
        kk = k.astype(np.int64)
        nz = gmax > 0
        # the smallest power of two whose 6 multiple holds the group maximum
        assert np.all(gmax[nz] <= 6 * np.ldexp(1.0, kk[nz]))
        assert np.all(gmax[nz] > 6 * np.ldexp(1.0, kk[nz] - 1))
        assert np.all(kk[~nz] == -126)
    assert np.all(dm[0, 0, 1, :32] == 0) and np.all(dv[1, 1, 2, 32:] == 0)
    assert np.all(qs["cv"] < 8)                 # variances carry no sign


def test_fp4_codes_are_the_nearest_e2m1_values():
    # brute force: every scaled value against all 15 distinct values; at an exact
    # midpoint the even mantissa (code bit 0 clear) wins
    rng = np.random.default_rng(81)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    y = np.concatenate([mids, -mids, rng.uniform(-6, 6, 2000)])
    y = y[: (len(y) // 32) * 32].reshape(1, 1, -1, 32)
    y[..., 0] = 6.0                             # every group's scale is 2^0
    qs = oracle.quantize_stats(y, np.zeros_like(y), "fp4")
    assert np.all(qs["km"] == 0)
    vals = np.array(E2M1_TABLE)
    for yy, c in zip(y.reshape(-1), qs["cm"].reshape(-1)):
        yy32 = float(np.float32(yy))
        dist = np.abs(abs(yy32) - vals)
        best = np.flatnonzero(dist == dist.min())
        want = best[0] if len(best) == 1 else best[best % 2 == 0][0]
        assert int(c) & 7 == want and (int(c) >> 3) == int(np.signbit(yy32))


def test_fp4_power_of_two_scaling_shifts_only_the_exponent():
    mean, var = _fp4_inputs(82)
    q0 = oracle.quantize_stats(mean, var, "fp4")
    q1 = oracle.quantize_stats(mean * 2.0 ** 7, var * 2.0 ** -5, "fp4")
    assert np.array_equal(q0["cm"], q1["cm"]) and np.array_equal(q0["cv"], q1["cv"])
    nzm = np.abs(mean).reshape(2, 2, 5, 2, 32).max(-1) > 0
    nzv = var.reshape(2, 2, 5, 2, 32).max(-1) > 0
    assert np.all(q1["km"][nzm].astype(int) == q0["km"][nzm].astype(int) + 7)
    assert np.all(q1["kv"][nzv].astype(int) == q0["kv"][nzv].astype(int) - 5)


def test_fp4_on_the_grid_round_trip_exactly():
    rng = np.random.default_rng(83)
    vals = np.array(E2M1_TABLE)
    m = vals[rng.integers(0, 8, (1, 2, 3, 64))] * rng.choice([-1.0, 1.0], (1, 2, 3, 64))
    m[..., 0] = 6.0                             # every group reaches the top value
    m[..., 32] = -6.0
    v = vals[rng.integers(0, 8, (1, 2, 3, 64))]
    v[..., 0] = 6.0
    v[..., 32] = 6.0
    mean, var = m * 2.0 ** -4, v * 2.0 ** 3
    qs = oracle.quantize_stats(mean, var, "fp4")
    dm, dv = oracle.dequantize_stats(qs)
    assert np.array_equal(dm, mean) and np.array_equal(dv, var)
    assert np.all(qs["km"] == -4) and np.all(qs["kv"] == 3)


def test_fp4_selection_equals_plain_selection_on_grid_statistics():
    # keys constant within a block, on the E2M1 grid: the mean is exactly
    # representable, the variance 0, so the selection is that of fp32 statistics
    rng = np.random.default_rng(84)
    B, Hq, Hkv, T, d, blk = 1, 4, 2, 256, 64, 32
    grid = np.array(E2M1_TABLE, np.float32) * np.float32(0.125)
    vals = grid[rng.integers(0, 8, (B, Hkv, T // blk, d))] * rng.choice([-1, 1], (B, Hkv, T // blk, d)).astype(np.float32)
    vals[..., 0] = 6 * 0.125
    vals[..., 32] = -6 * 0.125
    k = np.repeat(vals, blk, axis=2)
    q = _rand((B, Hq, T, d), 85)
    a = oracle.select(q, k, "f32", blk, 0.125, 0.6)
    b = oracle.select_quantized(q, k, "f32", blk, 0.125, 0.6, fmt="fp4")
    assert np.array_equal(a["count"], b["count"]) and np.array_equal(a["idx"], b["idx"])
    assert np.array_equal(a["scores"], b["scores"])


# ---------------------------------------------------------------- score-ordered early stop
# S2O, sections 2-3: blocks in descending estimated importance after the dense pass
# over the own block; stop once a block's marginal gain in attention mass falls
# below tau relative to the accumulated mass.

def _ordered_full_lists(B, Hq, T, blk):
    """Every causal block, in traversal order: own block, sink, then ascending."""
    nb = -(-T // blk)
    idx = np.full((B, Hq, nb, nb), -1, np.int32)
    cnt = np.zeros((B, Hq, nb), np.int32)
    for i in range(nb):
        order = [i] + ([0] if i > 0 else []) + list(range(1, i))
        idx[:, :, i, :len(order)] = order
        cnt[:, :, i] = len(order)
    return idx, cnt


def test_early_stop_constant_keys_closed_form():
    # k = 0: every logit is 0, so a block's gain for the row at offset r of query
    # block i is its number of visible tokens: r + 1 for the own block, blk for the
    # others. The tightest row is r = 0: after the own block, the sink and m more
    # blocks, its ratio is blk / (1 + (m + 1) blk). With blk = 4 the ratios of the
    # ranked blocks m = 1, 2, 3, ... are 4/9, 4/13, 4/17, 4/21: tau = 0.25 stops at
    # the third ranked block (4/17 < 0.25 <= 4/13), after 5 list entries.
    B, Hq, T, blk, d = 1, 2, 40, 4, 8
    q = _rand((B, Hq, T, d), 80)
    k = np.zeros((B, 1, T, d), np.float32)
    idx, cnt = _ordered_full_lists(B, Hq, T, blk)
    done, rat = oracle.early_stop(q, k, "f32", blk, idx, cnt, 0.125, 0.25)
    for i in range(T // blk):
        expect = 5 if i >= 5 else cnt[0, 0, i]
        assert np.all(done[:, :, i] == expect), (i, done[:, :, i], expect)
    np.testing.assert_allclose(rat[0, 0, 7, 2:5], [4 / 9, 4 / 13, 4 / 17], rtol=1e-14)
    assert rat[0, 0, 7, 5] == -1.0


def test_early_stop_limits_of_tau():
    B, Hq, Hkv, T, blk, d = 1, 4, 2, 48, 8, 8
    q, k = _rand((B, Hq, T, d), 81), _rand((B, Hkv, T, d), 82)
    idx, cnt = _ordered_full_lists(B, Hq, T, blk)
    done0, _ = oracle.early_stop(q, k, "f32", blk, idx, cnt, 0.3, 0.0)
    assert np.array_equal(done0, cnt)                  # a ratio is never below 0
    done1, _ = oracle.early_stop(q, k, "f32", blk, idx, cnt, 0.3, 1.5)
    reserved = np.minimum(cnt, 2)                      # own block + sink
    expect = np.where(cnt > reserved, reserved + 1, cnt)   # first ranked block: ratio <= 1
    assert np.array_equal(done1, expect)


def test_early_stop_ratio_is_gain_over_accumulated_mass():
    # two-block unit written out: own block then one ranked block, one row each
    B, Hq, T, blk, d = 1, 1, 4, 2, 1
    q = np.array([[[[0.0], [0.0], [1.0], [1.0]]]], np.float32)
    k = np.array([[[[0.0], [1.0], [2.0], [0.5]]]], np.float32)
    idx = np.array([[[[0, -1], [1, 0]]]], np.int32)
    cnt = np.array([[[1, 2]]], np.int32)
    _, rat = oracle.early_stop(q, k, "f32", blk, idx, cnt, 1.0, 0.0, n_sink=0, n_local=1)
    # query block 1, rows t = 2, 3 (q = 1): own block keys 2 (both rows) and 3 (row 3):
    # row 2: own gain e^2, then block 0 gain e^0 + e^1; row 3: own e^2 + e^0.5, then 1 + e.
    g_own = np.array([math.exp(2), math.exp(2) + math.exp(0.5)])
    g0 = np.array([1 + math.e, 1 + math.e])
    assert rat[0, 0, 1, 0] == pytest.approx(1.0)
    assert rat[0, 0, 1, 1] == pytest.approx(np.max(g0 / (g_own + g0)), rel=1e-14)


def test_score_order_lists_are_the_kept_sets_in_rank_order():
    B, Hq, Hkv, T, d, blk = 1, 4, 2, 96, 16, 8
    q, k = _rand((B, Hq, T, d), 83), _rand((B, Hkv, T, d), 84)
    sel = oracle.select(q, k, "f32", blk, 0.25, 0.6)
    oidx, ocnt = oracle.score_order(sel, T, T, blk)
    assert np.array_equal(ocnt, sel["count"])
    for (b, h, i), c in np.ndenumerate(ocnt):
        lst = oidx[b, h, i, :c].tolist()
        assert sorted(lst) == sel["idx"][b, h, i, :c].tolist()
        assert lst[0] == i                               # the own block first
        ranked = [j for j in lst if 1 <= j <= i - 1]
        if i > 0:
            assert lst[1] == 0                           # then the sink
        s32 = [float(np.float32(sel["scores"][b, h, i, j])) for j in ranked]
        assert all((s32[x], -ranked[x]) >= (s32[x + 1], -ranked[x + 1]) for x in range(len(s32) - 1))


def test_score_order_overlapping_sink_and_local_ranges():
    # S2O, section 2 (the dense local pass first) with SpotAttention's reserved
    # ranges: where the sink range [0, n_sink) and the local range [i - n_local + 1, i]
    # overlap, the overlap belongs to the sink, as in the cut. n_sink = n_local = 2,
    # full lists, worked out by hand: i = 0 -> [0]; i = 1 -> [0, 1] (block 1 lies in
    # the sink range); i = 2 -> [2, 0, 1]; i = 3 -> [3, 2, 0, 1]; i = 4 -> the local
    # blocks 4, 3, the sink 0, 1, then the ranked block 2.
    nq, blk = 5, 4
    idx, cnt = oracle.full_lists(1, 1, nq * blk, nq * blk, blk)
    l = np.zeros(idx.shape, np.float64)
    oi, oc = oracle.score_order({"idx": idx, "count": cnt, "scores": l}, nq * blk, nq * blk, blk,
                                n_sink=2, n_local=2)
    assert np.array_equal(oc, cnt)
    expect = [[0], [0, 1], [2, 0, 1], [3, 2, 0, 1], [4, 3, 0, 1, 2]]
    for i in range(nq):
        assert oi[0, 0, i, :cnt[0, 0, i]].tolist() == expect[i]


# ---------------------------------------------------------------- segmented key permutation
# PBS (Sparsere Blok-Sparse Attention via Tokenpermutatie), sections 2-3: keys sorted
# by global importance inside segments; segments keep their causal order.

def test_segperm_hand_worked_permutation():
    # Section 3 (proxy scoring): the mean-pooled softmax rows of the last query
    # block, worked out in closed form; the logit, unnormalised and first-block
    # readings each give another order on this input (derivation in the golden file).
    g = _golden()["segmented_permutation"]
    q = np.array(g["q"], np.float32)[None, None]
    k = np.array(g["k"], np.float32)[None, None]
    perm, imp = oracle.pbs_permutation(q, k, "f32", g["block"], g["seg_blocks"], g["scale"],
                                       return_importance=True)
    np.testing.assert_allclose(imp.reshape(-1), g["expected_importance"], rtol=1e-12, atol=0)
    assert perm.reshape(-1).tolist() == g["expected_perm"]


def _segperm_case(seed, L=90, blk=8, Hq=4, Hkv=2, d=8):
    # L = 90: the last query block is ragged (2 rows)
    return _rand((1, Hq, L, d), seed), _rand((1, Hkv, L, d), seed + 1), blk


def test_segperm_importance_sums_to_one_and_sorts_each_segment():
    # Every softmax row sums to 1, so their mean does too; each segment is a
    # permutation of its own keys, in descending importance (equal values: smaller
    # index first).
    q, k, blk = _segperm_case(90)
    seg = 3
    perm, imp = oracle.pbs_permutation(q, k, "f32", blk, seg, 0.4, return_importance=True)
    np.testing.assert_allclose(imp.sum(axis=-1), 1.0, rtol=1e-13)
    assert (imp >= 0).all()
    L, S = q.shape[2], seg * blk
    for g in range(k.shape[1]):
        i32 = imp[0, g].astype(np.float32)
        for s0 in range(0, L, S):
            p = perm[0, g, s0:s0 + S]
            assert sorted(p.tolist()) == list(range(s0, min(s0 + S, L)))
            assert all((i32[p[x]], -p[x]) >= (i32[p[x + 1]], -p[x + 1]) for x in range(len(p) - 1))


def test_segperm_importance_at_vanishing_scale_is_uniform_causal():
    # As s -> 0 every causal row is uniform over keys 0..t: importance(u) =
    # (1 / n_rows) sum over the last block's rows t >= u of 1 / (t + 1), the same for
    # every head. Pins the causal limit and which rows are pooled.
    q, k, blk = _segperm_case(92)
    L = q.shape[2]
    _, imp = oracle.pbs_permutation(q, k, "f32", blk, 2, 1e-12, return_importance=True)
    r0 = (-(-L // blk) - 1) * blk
    rows = np.arange(r0, L)
    ref = np.array([sum(1.0 / (t + 1) for t in rows if t >= u) for u in range(L)]) / rows.size
    np.testing.assert_allclose(imp[0, 0], ref, rtol=1e-9, atol=1e-15)
    np.testing.assert_allclose(imp[0, 1], ref, rtol=1e-9, atol=1e-15)


def test_segperm_importance_invariant_to_a_per_row_logit_offset():
    # A key component shared by every key adds q_t[c] to each logit of row t: the
    # softmax of the row, and so the importance, does not change.
    q, k, blk = _segperm_case(94)
    k[..., -1] = 1.0
    q2 = q.copy()
    L = q.shape[2]
    r0 = (-(-L // blk) - 1) * blk
    q2[:, :, r0:, -1] += np.float32(3.0) * np.arange(1, q.shape[1] * (L - r0) + 1,
                                                        dtype=np.float32).reshape(q.shape[1], -1)[None]
    _, a = oracle.pbs_permutation(q, k, "f32", blk, 2, 0.5, return_importance=True)
    _, b = oracle.pbs_permutation(q2, k, "f32", blk, 2, 0.5, return_importance=True)
    np.testing.assert_allclose(b, a, rtol=1e-10, atol=1e-15)


def test_segperm_importance_reads_only_its_groups_last_block():
    # kv-group 0 pools heads 0 and 1 (G = 2), over the rows of the last query block
    # only: queries of the other group, or of earlier rows, change nothing.
    q, k, blk = _segperm_case(96)
    L = q.shape[2]
    r0 = (-(-L // blk) - 1) * blk
    _, a = oracle.pbs_permutation(q, k, "f32", blk, 2, 0.5, return_importance=True)
    q2 = q.copy()
    q2[:, 2:] = _rand(q2[:, 2:].shape, 97)          # the other group's heads
    q2[:, :2, :r0] = _rand(q2[:, :2, :r0].shape, 98)  # earlier rows of this group
    _, b = oracle.pbs_permutation(q2, k, "f32", blk, 2, 0.5, return_importance=True)
    np.testing.assert_array_equal(b[0, 0], a[0, 0])
    q3 = q.copy()
    q3[:, 1, L - 1] += 1.0                          # a last-block row of head 1
    _, c = oracle.pbs_permutation(q3, k, "f32", blk, 2, 0.5, return_importance=True)
    assert not np.allclose(c[0, 0], a[0, 0], rtol=1e-6, atol=0)
    np.testing.assert_array_equal(c[0, 1], a[0, 1])


def test_segperm_at_p_one_is_dense_causal_attention():
    B, Hq, Hkv, L, d, blk = 1, 4, 2, 64, 16, 8
    q, k, v = _rand((B, Hq, L, d), 92), _rand((B, Hkv, L, d), 93), _rand((B, Hkv, L, d), 94)
    ref = _dense_causal_numpy(q, k, v, 0.25)
    for seg in (1, 2, 3):
        sel = oracle.select_segperm(q, k, "f32", blk, seg, 0.25, 1.0)
        out, _ = oracle.attention_segperm(q, k, v, "f32", blk, seg, sel["perm"], sel["idx"],
                                          sel["count"], 0.25)
        np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-12)


def test_segperm_with_one_segment_is_the_plain_path():
    B, Hq, Hkv, L, d, blk = 1, 4, 2, 64, 16, 8
    q, k, v = _rand((B, Hq, L, d), 95), _rand((B, Hkv, L, d), 96), _rand((B, Hkv, L, d), 97)
    a = oracle.select(q, k, "f32", blk, 0.25, 0.6)
    b = oracle.select_segperm(q, k, "f32", blk, 8, 0.25, 0.6)     # 8 blocks: one segment
    assert np.array_equal(a["idx"], b["idx"]) and np.array_equal(a["count"], b["count"])
    oa, _ = oracle.attention(q, k, v, "f32", blk, a["idx"], a["count"], 0.25)
    ob, _ = oracle.attention_segperm(q, k, v, "f32", blk, 8, b["perm"], b["idx"], b["count"], 0.25)
    np.testing.assert_allclose(ob, oa, rtol=1e-13, atol=1e-14)


def test_segperm_attention_in_the_permuted_layout():
    # The same masked attention evaluated directly on the permuted keys: earlier
    # segments by permuted block, the own segment in original order and causal.
    B, Hq, Hkv, L, d, blk, seg = 1, 2, 1, 48, 8, 4, 3
    q, k, v = _rand((B, Hq, L, d), 98), _rand((B, Hkv, L, d), 99), _rand((B, Hkv, L, d), 100)
    sel = oracle.select_segperm(q, k, "f32", blk, seg, 0.5, 0.5)
    perm = sel["perm"]
    out, _ = oracle.attention_segperm(q, k, v, "f32", blk, seg, perm, sel["idx"], sel["count"], 0.5)
    kp, vp = oracle.permute(k, perm)[0, 0].astype(np.float64), oracle.permute(v, perm)[0, 0].astype(np.float64)
    ko, vo = k[0, 0].astype(np.float64), v[0, 0].astype(np.float64)
    for h in range(Hq):
        for t in range(L):
            i = t // blk
            s0 = (i // seg) * seg * blk
            kept = set(sel["idx"][0, h, i, :sel["count"][0, h, i]].tolist())
            keys, vals = [], []
            for p in range(s0):                      # earlier segments, permuted layout
                if p // blk in kept:
                    keys.append(kp[p]); vals.append(vp[p])
            for u in range(s0, t + 1):               # own segment, original layout
                if u // blk in kept:
                    keys.append(ko[u]); vals.append(vo[u])
            z = 0.5 * np.array(keys) @ q[0, h, t].astype(np.float64)
            w = np.exp(z - z.max())
            np.testing.assert_allclose(out[0, h, t], (w / w.sum()) @ np.array(vals), rtol=1e-11,
                                       atol=1e-12)
