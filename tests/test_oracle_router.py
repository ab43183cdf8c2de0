"""Pins for the oracle's router, top-k selection, weights and bucketing.

Sources: "GLM-5.2-colibri-int4架构解析…" (wmrh.cn), sections "MoE的工作原理"
(each token's router scores pick the best 8 experts; their outputs are summed
weighted by the scores) and "高级配置选项 / 路由策略定制" (topk_method,
routed_scaling_factor, norm_topk_prob); "Colibri：在笔记本上跑744B参数的AI
模型", "关键特性" (DeepSeek-V3 style sigmoid router); "如何在普通电脑上运行
7440 亿参数神经网络", "引擎是如何工作的" (requests for one expert merged into
one batch).  Correction bias, ties to the lower index and the order of the
weight arithmetic are the readings stated in the design notes."""
import itertools
from fractions import Fraction

import numpy as np
import pytest

U = 2.0 ** -24


def _tiny(syn):
    cfg = syn.config("tiny")
    return cfg, syn.router_w(cfg), syn.bias(cfg), syn.tokens(cfg)


def test_logit_within_error_bound_of_exact(ora, syn):
    cfg, W, _, x = _tiny(syn)
    for H in (128, 256):
        for t in range(x.shape[0]):
            for e in range(W.shape[0]):
                got = ora.router_logit(x[t, :H], W[e, :H])
                xs = [Fraction(float(v)) for v in x[t, :H]]
                ws = [Fraction(float(v)) for v in W[e, :H]]
                exact = sum(a * b for a, b in zip(xs, ws))
                mag = sum(abs(a * b) for a, b in zip(xs, ws))
                # each accumulator: H/128 fmas; then 31 adds
                gamma = (H // 128 + 32) * U
                assert abs(Fraction(got) - exact) <= Fraction(gamma) * mag * 1.01


def test_logit_glm_row_against_double(ora, syn):
    cfg = syn.config("decode1")
    W = syn.normal(4 * 6144, 0, 0, syn.TID_ROUTER, cfg["sigma_router"]).reshape(4, 6144)
    x = syn.tokens(cfg)[0]
    for e in range(4):
        got = ora.router_logit(x, W[e])
        prod = x.astype(np.float64) * W[e].astype(np.float64)
        assert abs(got - prod.sum()) <= (6144 // 128 + 32) * U * np.abs(prod).sum()


def test_scores_are_sigmoid_of_logits(ora, syn):
    cfg, W, b, x = _tiny(syn)
    s, _, _ = ora.route(x, W, b, 4, True, 2.5)
    for t in range(x.shape[0]):
        for e in range(W.shape[0]):
            assert s[t, e] == np.float32(ora.sigmoid(ora.router_logit(x[t], W[e])))


def _exhaustive_choice(bvals, K):
    fr = [Fraction(float(v)) for v in bvals]
    best, best_sets = None, []
    for sub in itertools.combinations(range(len(bvals)), K):
        s = sum(fr[i] for i in sub)
        if best is None or s > best:
            best, best_sets = s, [sub]
        elif s == best:
            best_sets.append(sub)
    return min(best_sets)  # lexicographically lowest index set among the maximisers


def test_topk_exhaustive_tiny(ora, syn):
    cfg, W, b, x = _tiny(syn)
    s, idx, _ = ora.route(x, W, b, 4, True, 2.5)
    for t in range(x.shape[0]):
        bt = (s[t] + b).astype(np.float32)
        assert tuple(sorted(idx[t])) == _exhaustive_choice(bt, 4)
        # rank order: descending biased score, ties to the lower index
        vals = [(-float(bt[e]), int(e)) for e in idx[t]]
        assert vals == sorted(vals)


def test_topk_ties_go_to_lower_index(ora):
    # zero router: every score is sigmoid(0) = 0.5; the bias alone decides,
    # with deliberate exact ties.
    E, H, K = 16, 128, 4
    W = np.zeros((E, H), np.float32)
    x = np.ones((3, H), np.float32)
    bias = np.zeros(E, np.float32)
    bias[[3, 9, 12]] = 0.25
    bias[[5, 14]] = 0.125
    s, idx, w = ora.route(x, W, bias, K, True, 2.5)
    assert np.all(s == 0.5)
    for t in range(3):
        assert list(idx[t]) == [3, 9, 12, 5]
        assert tuple(sorted(idx[t])) == _exhaustive_choice((s[t] + bias).astype(np.float32), K)
    _, idx1, _ = ora.route(x, W, np.zeros(E, np.float32), K, True, 2.5)
    assert list(idx1[0]) == [0, 1, 2, 3]


def test_bias_selects_but_does_not_weight(ora, syn):
    cfg, W, b, x = _tiny(syn)
    s, idx, w = ora.route(x, W, b, 4, False, 1.0)
    for t in range(x.shape[0]):
        assert np.array_equal(w[t], s[t, idx[t]])  # weights from the unbiased score


def test_k_equals_e_selects_everything_in_rank_order(ora, syn):
    cfg, W, b, x = _tiny(syn)
    E = W.shape[0]
    s, idx, _ = ora.route(x, W, b, E, True, 2.5)
    for t in range(x.shape[0]):
        bt = (s[t] + b).astype(np.float32)
        want = np.lexsort((np.arange(E), -bt.astype(np.float64)))
        assert np.array_equal(idx[t], want)


@pytest.mark.parametrize("rsf", [2.5, 1.0, 0.75])
def test_normalised_weights_sum_to_rsf(ora, syn, rsf):
    cfg = syn.config("decode16")
    W, b, x = syn.router_w(cfg), syn.bias(cfg), syn.tokens(cfg)
    s, idx, w = ora.route(x, W, b, 8, True, rsf)
    for t in range(x.shape[0]):
        tot = float(np.sum(w[t].astype(np.float64)))
        assert abs(tot - rsf) <= 8 * 4 * U * rsf
        ratio = w[t].astype(np.float64) / s[t, idx[t]].astype(np.float64)
        assert np.ptp(ratio) <= 4 * U * ratio.mean()
        # descending biased score
        bt = (s[t, idx[t]] + b[idx[t]]).astype(np.float32)
        assert np.all(np.diff(bt.astype(np.float64)) <= 0)


def test_unnormalised_weights_are_scaled_scores(ora, syn):
    cfg, W, b, x = _tiny(syn)
    s, idx, w = ora.route(x, W, b, 4, False, 2.5)
    for t in range(x.shape[0]):
        assert np.array_equal(w[t], (s[t, idx[t]] * np.float32(2.5)).astype(np.float32))


# --------------------------------------------------------------------------
# bucketing

def _bucket_ref(idx, E):
    T, K = idx.shape
    flat = idx.ravel()
    counts = np.bincount(flat, minlength=E)
    key = flat.astype(np.int64) * T + np.repeat(np.arange(T), K)
    perm = np.argsort(key, kind="stable")
    return counts, perm


@pytest.mark.parametrize("T,K,E", [(8, 4, 16), (1, 8, 256), (16, 8, 256), (300, 8, 256), (5, 16, 16)])
def test_bucket_matches_sort(ora, T, K, E):
    rng = np.random.default_rng(T * 1000 + K)
    idx = np.stack([rng.permutation(E)[:K] for _ in range(T)]).astype(np.int32)
    counts, offsets, perm = ora.bucket(idx, E)
    c_ref, p_ref = _bucket_ref(idx, E)
    assert np.array_equal(counts, c_ref)
    assert offsets[0] == 0 and offsets[-1] == T * K
    assert np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(perm, p_ref)
    # every pair appears once, and each group holds only its expert
    assert np.array_equal(np.sort(perm), np.arange(T * K))
    for e in range(E):
        grp = perm[offsets[e]:offsets[e + 1]]
        assert np.all(idx.ravel()[grp] == e)
        assert np.all(np.diff(grp // K) > 0)


def test_bucket_empty(ora):
    counts, offsets, perm = ora.bucket(np.zeros((0, 8), np.int32), 256)
    assert np.all(counts == 0) and np.all(offsets == 0) and perm.size == 0
