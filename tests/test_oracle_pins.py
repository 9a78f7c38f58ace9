"""Pins of the CPU oracle to things other than itself.

Each test checks the oracle against a value the pages print, a hand
enumeration, brute-force loops written independently here, a library
routine, or an invariant the method guarantees.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import ai_oracle as O
from synth import workloads as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- scoring --

def test_worked_example_mean_rep_hides_member():
    """Explainer, 代表向量为什么要学？ box: members -2 and 2, query 1, one head
    of weight 1: the mean representative scores 0, the members 0 and 2."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    keys = np.array(g["members"]).reshape(-1, 1)
    q = np.array([[g["query"]]])
    w = np.array([g["weight"]])
    mean = keys.mean(0, keepdims=True)
    assert mean[0, 0] == g["mean_representative"]
    assert O.indexer_score(q, w, mean)[0] == g["representative_score"]
    ms = O.indexer_score(q, w, keys)
    assert ms.tolist() == g["member_scores"]
    assert ms.mean() == g["member_score_mean"]
    ids, _ = O.exhaustive_select(q, w, keys, t=1, k=1)
    assert ids.tolist() == [g["should_select_member"]]


def _score_loops(q, w, keys):
    out = []
    for s in range(keys.shape[0]):
        tot = 0.0
        for h in range(q.shape[0]):
            dot = 0.0
            for i in range(q.shape[1]):
                dot += q[h, i] * keys[s, i]
            tot += w[h] * (dot if dot > 0 else 0.0)
        out.append(tot)
    return np.array(out)


def test_indexer_score_matches_loops():
    g = np.random.default_rng(1)
    q = g.standard_normal((3, 5))
    w = g.standard_normal(3)
    keys = g.standard_normal((40, 5))
    np.testing.assert_allclose(O.indexer_score(q, w, keys), _score_loops(q, w, keys),
                               rtol=1e-12, atol=1e-12)


def test_inner_product_identity_without_relu():
    """Explainer, 代表向量为什么要学？: with plain inner products the mean is an
    exact representative; with every q_h.k >= 0 the ReLU is inactive and
    I(q, mean) equals the mean member score."""
    g = np.random.default_rng(2)
    q = np.abs(g.standard_normal((4, 6)))
    keys = np.abs(g.standard_normal((9, 6)))
    w = g.standard_normal(4)
    lhs = O.indexer_score(q, w, keys.mean(0, keepdims=True))[0]
    rhs = O.indexer_score(q, w, keys).mean()
    assert math.isclose(lhs, rhs, rel_tol=1e-12, abs_tol=1e-12)
    # and with mixed signs the identity fails (the box's point)
    keys2 = np.array([[-2.0], [2.0]])
    assert O.indexer_score(np.ones((1, 1)), np.ones(1), keys2.mean(0, keepdims=True))[0] \
        < O.indexer_score(np.ones((1, 1)), np.ones(1), keys2).mean()


def test_head_weights_sign_and_relu_order():
    # one head with negative weight: ReLU applies to the dot, then the weight
    q = np.array([[1.0, 0.0], [0.0, 1.0]])
    w = np.array([2.0, -3.0])
    keys = np.array([[1.0, 1.0], [-1.0, 2.0], [3.0, -1.0]])
    assert O.indexer_score(q, w, keys).tolist() == [2 - 3, 0 - 6, 6 - 0]


# ------------------------------------------------------------------ top-k --

def test_topk_tie_break_and_padding():
    scores = np.array([1.0, 3.0, 3.0, 2.0, 3.0])
    ids = np.array([10, 4, 7, 1, 2])
    out, sc = O.topk_ids(scores, ids, 4)
    assert out.tolist() == [2, 4, 7, 1]
    out, _ = O.topk_ids(scores, ids, 7)
    assert out.tolist() == [2, 4, 7, 1, 10, -1, -1]


def test_exhaustive_matches_bruteforce():
    g = np.random.default_rng(3)
    L, d, H = 48, 6, 3
    keys = g.standard_normal((L, d))
    for t in [0, 1, 7, 30, 47]:
        q = g.standard_normal((H, d))
        w = g.standard_normal(H)
        sc = _score_loops(q, w, keys[:t + 1])
        pairs = sorted(((-sc[s], s) for s in range(t + 1)))
        want = [s for _, s in pairs[:5]] + [-1] * max(0, 5 - (t + 1))
        got, _ = O.exhaustive_select(q, w, keys, t, 5)
        assert got.tolist() == want


# ---------------------------------------------------------------- formats --

def test_bf16_rne_matches_torch():
    g = np.random.default_rng(4)
    x = np.concatenate([g.standard_normal(20000) * 10.0,
                        g.standard_normal(2000) * 1e-3])
    x32 = x.astype(np.float32).astype(np.float64)  # values torch can hold exactly
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16_rne(x32), want)
    # ties to even: 1 + 2^-8 is halfway between 1 and 1 + 2^-7
    assert O.bf16_rne(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    assert O.bf16_rne(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


def test_e4m3_rne_matches_torch_in_range():
    g = np.random.default_rng(5)
    x = np.concatenate([g.uniform(-448, 448, 20000), g.standard_normal(20000),
                        g.standard_normal(2000) * 1e-2]).astype(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.e4m3_rne(x), want)
    # saturation (definition): beyond the largest finite value -> +-448
    assert O.e4m3_rne(np.array([500.0, -1e6], dtype=np.float32)).tolist() == [448.0, -448.0]
    # smallest subnormal 2^-9, and halfway below it rounds to zero (even)
    assert O.e4m3_rne(np.array([2.0 ** -9, 2.0 ** -10], dtype=np.float32)).tolist() == [2.0 ** -9, 0.0]


def test_fp8_quantize_scale_is_amax_over_448():
    g = np.random.default_rng(6)
    k = g.standard_normal((50, 16)).astype(np.float32)
    codes, scale = O.quantize_fp8_keys(k)
    np.testing.assert_array_equal(scale, (np.abs(k).max(1) / np.float32(448)).astype(np.float32))
    assert np.abs(codes).max() <= 448
    # every row's largest magnitude maps to (about) 448
    assert np.all(np.abs(codes).max(1) >= 416)
    # dequantized keys are close: e4m3 has relative spacing 2^-3
    deq = codes * scale[:, None]
    assert np.all(np.abs(deq - k) <= np.abs(k) * 2.0 ** -4 + scale[:, None] * 2.0 ** -9)


# ------------------------------------------------------------------- seal --

def test_seal_hand_enumeration_capacity_binds():
    """1-D window X = [0,1,2,3,10,11], m = 2, cap = 3, by hand:
    init c = (X[1], X[4]) = (1, 10).  Pairs by (D, i, j): (0:1,0) (0:4,1)
    (1:0,0) (1:2,0) (1:5,1) (4:3,0) -> cluster 0 is full, so key 3 waits
    for (49:3,1).  Assignment [0,0,0,1,1,1], centres (1, 8).  The second
    pass repeats the assignment and stops."""
    X = np.array([0.0, 1.0, 2.0, 3.0, 10.0, 11.0]).reshape(-1, 1)
    assign, C = O.seal_window(X, m=2, cap=3, iters=10)
    assert assign.tolist() == [0, 0, 0, 1, 1, 1]
    assert C.ravel().tolist() == [1.0, 8.0]
    # without the cap key 3 would join cluster 0
    assign, C = O.seal_window(X, m=2, cap=6, iters=10)
    assert assign.tolist() == [0, 0, 0, 0, 1, 1]
    assert C.ravel().tolist() == [1.5, 10.5]


def _greedy_loops(X, C, cap):
    pairs = []
    for i in range(X.shape[0]):
        for j in range(C.shape[0]):
            dist = sum((X[i, a] - C[j, a]) ** 2 for a in range(X.shape[1]))
            pairs.append((dist, i, j))
    pairs.sort()
    assign = [-1] * X.shape[0]
    count = [0] * C.shape[0]
    for _, i, j in pairs:
        if assign[i] < 0 and count[j] < cap:
            assign[i] = j
            count[j] += 1
    return assign


def test_seal_one_iteration_matches_loops():
    g = np.random.default_rng(7)
    X = g.standard_normal((24, 3))
    m, cap = 4, 6
    assign, C = O.seal_window(X, m=m, cap=cap, iters=1)
    C0 = np.stack([X[((2 * j + 1) * 24) // (2 * m)] for j in range(m)])
    assert assign.tolist() == _greedy_loops(X, C0, cap)
    for j in range(m):
        np.testing.assert_allclose(C[j], X[assign == j].mean(0), rtol=0, atol=1e-15)


def test_seal_invariants_random():
    g = np.random.default_rng(8)
    X = g.standard_normal((256, 8)) + 3 * g.standard_normal((1, 8))
    assign, C = O.seal_window(X, m=8, cap=32, iters=10)
    counts = np.bincount(assign, minlength=8)
    assert counts.sum() == 256 and counts.max() <= 32
    for j in range(8):
        np.testing.assert_allclose(C[j], X[assign == j].mean(0), atol=1e-14)


# ------------------------------------------------------------------ refit --

def test_splitmix64_published_first_output():
    # SplitMix64 from state 0: first output 0xE220A8397B1DCDAF
    assert O.splitmix64(0, 0) == 0xE220A8397B1DCDAF


def test_refit_seed_ids_distinct_in_range_and_uniform():
    ids = O.refit_seed_ids(0, 3, 100, 164, 64)
    assert sorted(ids.tolist()) == list(range(100, 164))   # all of a full window
    counts = np.zeros(50)
    for r in range(400):
        s = O.refit_seed_ids(7, r, 0, 50, 5)
        assert len(set(s.tolist())) == 5 and s.min() >= 0 and s.max() < 50
        counts[s] += 1
    # 2000 draws over 50 ids: each ~40; a biased sampler would be far off
    assert counts.min() > 15 and counts.max() < 70


def test_refit_lloyd_matches_loops():
    g = np.random.default_rng(9)
    X = g.standard_normal((60, 4))
    C0 = g.standard_normal((7, 4))
    C0[5] = 50.0  # a centre nobody picks stays where it is
    assign, C = O.refit_lloyd(X, C0)
    for i in range(60):
        d = [sum((X[i, a] - C0[j, a]) ** 2 for a in range(4)) for j in range(7)]
        assert assign[i] == int(np.argmin(d))
    for j in range(7):
        if (assign == j).any():
            np.testing.assert_allclose(C[j], X[assign == j].mean(0), atol=1e-14)
        else:
            np.testing.assert_array_equal(C[j], C0[j])


def test_refit_tie_goes_to_lower_centre():
    X = np.array([[0.0, 0.0]])
    C0 = np.array([[1.0, 0.0], [-1.0, 0.0]])
    assign, _ = O.refit_lloyd(X, C0)
    assert assign.tolist() == [0]


# ---------------------------------------------------------------- encoder --

def test_encoder_zero_output_is_plain_ivf_and_bound_holds():
    wl = S.scaled(S.WORKLOADS["glm_bf16_L128k"], d=16, H=2)
    g = np.random.default_rng(10)
    members = g.standard_normal((30, 16))
    mu = members.mean(0)
    zero = S.encoder_weights(wl, zero_out=True)
    assert np.all(O.encoder_correction(members, mu, zero) == 0.0)
    rnd = S.encoder_weights(wl)
    corr = O.encoder_correction(members, mu, rnd)
    assert np.linalg.norm(corr) <= 0.25 * np.linalg.norm(mu) * (1 + 1e-12)
    assert np.linalg.norm(corr) > 0


def _enc(A, a, B1, b1, B2, b2):
    f = lambda x: np.asarray(x, dtype=np.float64)
    return {"A": f(A), "a": f(a), "B1": f(B1), "b1": f(b1), "B2": f(B2), "b2": f(b2)}


def _sel(i, n=7):
    e = np.zeros(n)
    e[i] = 1.0
    return e


def test_encoder_closed_forms():
    """Weights chosen so each stage of the correction reduces to numbers a
    reader can derive by hand (d = 2, so f has 3d + 1 = 7 entries in the
    order [mean phi ; max phi ; mu ; ln n]).  A swapped feature block, a
    missing ReLU or bias, or a wrong bound rule changes the result."""
    # 1. phi = ReLU(k); h picks max phi_0 and ln n; bound inactive, corr = t
    members = np.array([[1.0, 0.0], [3.0, 2.0]])
    mu = members.mean(0)                                   # [2, 1]
    w = _enc(np.eye(2), [0, 0], np.stack([_sel(2), _sel(6)]), [0, 0],
             [[0.1, 0.0], [0.0, 1.0]], [0.0, -0.5])
    # h = [max phi_0, ln 2] = [3, ln 2]; z = [0.3, ln 2 - 0.5]
    want = np.array([math.tanh(0.3), math.tanh(math.log(2.0) - 0.5)])
    assert np.linalg.norm(want) < 0.25 * math.sqrt(5.0)     # the bound does not bind
    np.testing.assert_allclose(O.encoder_correction(members, mu, w), want, rtol=0, atol=1e-15)
    # 2. the bound binds: corr = t * 0.25 ||mu|| / ||t|| = [0.25 * 0.2, 0]
    members = np.array([[0.2, 0.0], [-0.2, 0.4]])
    mu = members.mean(0)                                   # [0, 0.2]
    w = _enc(np.eye(2), [0, 0], np.zeros((2, 7)), [0, 0], np.zeros((2, 2)), [1.0, 0.0])
    np.testing.assert_allclose(O.encoder_correction(members, mu, w), [0.05, 0.0], rtol=0, atol=1e-15)
    # 3. phi = ReLU(k + a) with a = [-1, 0] clips; h picks mean phi_0 and max phi_1
    members = np.array([[0.5, -1.0], [2.0, 3.0]])
    mu = members.mean(0)                                   # [1.25, 1]
    w = _enc(np.eye(2), [-1.0, 0.0], np.stack([_sel(0), _sel(3)]), [0, 0], 0.2 * np.eye(2), [0, 0])
    # phi = [[0, 0], [1, 3]]: mean phi_0 = 0.5, max phi_1 = 3; z = 0.2 * [0.5, 3]
    t = np.array([math.tanh(0.1), math.tanh(0.6)])
    bound = 0.25 * math.hypot(1.25, 1.0)
    assert np.linalg.norm(t) > bound                       # the bound binds
    np.testing.assert_allclose(O.encoder_correction(members, mu, w), t * bound / np.linalg.norm(t),
                               rtol=1e-14, atol=0)
    # 4. a ReLU in h: a negative pre-activation gives h = 0, so t = tanh(b2)
    w = _enc(np.eye(2), [0, 0], np.stack([-_sel(2), -_sel(6)]), [0, 0], np.eye(2), [0.01, 0.0])
    members = np.array([[1.0, 0.0], [3.0, 2.0]])
    np.testing.assert_allclose(O.encoder_correction(members, members.mean(0), w),
                               [math.tanh(0.01), 0.0], rtol=0, atol=1e-15)


# ------------------------------------------------------------ index-level --

def _tiny_index(wl, enc=None):
    return O.OracleIndex(d=wl.d, n_sinks=wl.n_sinks, window=wl.window,
                         clusters_per_window=wl.clusters_per_window,
                         refit_period=wl.refit_period, seal_iters=wl.seal_iters,
                         seed=wl.seed, encoder=enc)


TINY = S.scaled(S.WORKLOADS["tiny_fp32_L4k"], L=1024, T=128, window=64, refit_period=256,
                budget=160, k=16, d=8, H=2, M=16)


def _run_prefill(wl, budget, enc=None):
    keys = S.keys_f64(wl).astype(np.float32).astype(np.float64)
    idx = _tiny_index(wl, enc)
    out = []
    for c in range(wl.n_chunks):
        p0 = c * wl.T
        idx.append(keys[p0:p0 + wl.T])
        idx.seal()
        q, w = S.queries_f64(wl, p0, p0 + wl.T)
        q = q.astype(np.float32).astype(np.float64)
        for i in range(wl.T):
            t = p0 + i
            cand, _, v = idx.candidates(t, q[i], w[i], budget)
            ids, _ = idx.route_refine(q[i], w[i], t, wl.k, budget)
            exh, _ = idx.exhaustive(q[i], w[i], t, wl.k)
            out.append((t, cand, v, ids, exh, idx))
    return idx, out


def test_budget_at_least_prefix_gives_exhaustive():
    _, rows = _run_prefill(TINY, budget=TINY.L)
    for t, cand, v, ids, exh, _ in rows:
        assert sorted(cand.tolist()) == list(range(t + 1))
        assert ids.tolist() == exh.tolist()


def test_causality_open_window_and_first_seal():
    idx, rows = _run_prefill(TINY, budget=TINY.budget)
    S0, W = TINY.n_sinks, TINY.window
    for t, cand, v, ids, exh, _ in rows:
        assert cand.max() <= t and ids.max() <= t               # no look-ahead
        assert v.n_clusters == 0 or v.n_v <= t + 1
        assert len(set(cand.tolist())) == cand.size             # no duplicates
        # open-window keys are candidates immediately (budget >= S + W here)
        assert set(range(v.n_v, t + 1)) <= set(cand.tolist())
        if t + 1 < S0 + W:                                       # before first seal
            assert ids.tolist() == exh.tolist()
    # every visible cluster of every version holds only keys below its watermark
    for v in idx.versions:
        for c in idx.clusters[:v.n_clusters]:
            assert c.members.size == 0 or c.members.max() < v.n_v
    ns = [v.n_v for v in idx.versions]
    assert ns == sorted(ns)


def test_clusters_partition_clustered_prefix_after_refit():
    idx, _ = _run_prefill(TINY, budget=TINY.budget)
    idx.publish()
    last = idx.versions[-1]
    mem = np.concatenate([c.members for c in idx.clusters[:last.n_clusters]])
    assert sorted(mem.tolist()) == list(range(TINY.n_sinks, last.n_v))
    assert idx.n_refits == (TINY.L - TINY.n_sinks) // TINY.refit_period


def test_zero_correction_reproduces_plain_ivf():
    wl = TINY
    enc = S.encoder_weights(S.scaled(wl), zero_out=True)
    _, plain = _run_prefill(wl, budget=wl.budget)
    _, zero = _run_prefill(wl, budget=wl.budget, enc=enc)
    for a, b in zip(plain, zero):
        assert a[1].tolist() == b[1].tolist() and a[3].tolist() == b[3].tolist()


def test_recall_definition():
    a = np.array([[1, 2, 3, -1], [4, 5, 6, 7]])
    b = np.array([[3, 2, 9, -1], [7, 6, 5, 4]])
    assert O.recall(a, a) == 1.0
    assert O.recall(b, a) == (2 + 4) / 7


# ------------------------------------------------- candidate fill, by hand --

def _hand_index():
    """A hand-built index state (explainer, 查询时怎么挑候选？ and the version
    paragraph of 索引怎么边算边建？), S = 4 sinks, 15 keys (ids 0..14).

    Window 1 = keys [4, 8) sealed into clusters c0, c1 -> version (2, 8).
    Window 2 = keys [8, 12) sealed into c2 (empty), c3, c4 -> version (5, 12).
    One head, weight 1, query q = (2, 1); route score = ReLU(2 r0 + r1):

      cluster  rep          score  members
      c0       (0.5, 0)     1.0    4, 6
      c1       (1.0, 0.5)   2.5    5, 7
      c2       (2, 2)       6.0    (empty: skipped)
      c3       (0.25, 0.5)  1.0    8, 10, 11   (ties c0: lower id first)
      c4       (-1, 0)      0.0    9
    """
    idx = O.OracleIndex(d=2, n_sinks=4, window=4, clusters_per_window=2, refit_period=0)
    idx.keys = np.zeros((15, 2))
    spec = [((0.5, 0.0), [4, 6]), ((1.0, 0.5), [5, 7]), ((2.0, 2.0), []),
            ((0.25, 0.5), [8, 10, 11]), ((-1.0, 0.0), [9])]
    idx.clusters = [O.Cluster(centroid=np.array(r), members=np.array(m, dtype=np.int64),
                              rep=np.array(r)) for r, m in spec]
    idx.versions = [O.Version(2, 8), O.Version(5, 12)]
    return idx, np.array([[2.0, 1.0]]), np.array([1.0])


@pytest.mark.parametrize("t,C,want", [
    # t = 14 uses version (5, 12): sinks, open window 12..14, then
    # c1 (2.5), c0 (1.0), c3 (1.0, tie -> after c0), c4 (0.0); c2 is empty
    (14, 100, [0, 1, 2, 3, 12, 13, 14, 5, 7, 4, 6, 8, 10, 11, 9]),
    (14, 10, [0, 1, 2, 3, 12, 13, 14, 5, 7, 4]),            # rank-2 list cut after one member
    (14, 13, [0, 1, 2, 3, 12, 13, 14, 5, 7, 4, 6, 8, 10]),  # tie order, rank-3 list cut
    (14, 5, [0, 1, 2, 3, 12]),                               # budget inside the open window
    # t = 10 uses version (2, 8) (watermark 12 > t + 1): open window 8..10,
    # only c1 and c0 visible
    (10, 100, [0, 1, 2, 3, 8, 9, 10, 5, 7, 4, 6]),
    (10, 9, [0, 1, 2, 3, 8, 9, 10, 5, 7]),
    # t = 2: no sealed version yet, sinks cut at t
    (2, 100, [0, 1, 2]),
])
def test_candidate_fill_order_by_hand(t, C, want):
    """The exact candidate sequence: sinks, open window ascending, member
    lists in rank order (score desc, cluster id asc) in CSR order, the last
    list truncated at C, empty clusters contributing nothing, clusters of
    newer versions invisible."""
    idx, q, w = _hand_index()
    cand, sc, v = idx.candidates(t, q, w, C)
    assert cand.tolist() == want
    if t >= 11:
        assert sc.tolist() == [1.0, 2.5, 6.0, 1.0, 0.0]
    # route+refine on this state returns ids drawn from exactly that list
    ids, _ = idx.route_refine(q, w, t, k=len(want), C=C)
    assert sorted(ids[ids >= 0].tolist()) == sorted(want)


def test_block_seal_by_hand():
    """Contiguous-block baseline (explainer, 它到底在解决什么问题？: HiSA groups
    keys by position): a window of 10 one-dimensional keys cut into m = 3
    blocks of consecutive keys, [0, 3), [3, 6), [6, 10), each represented by
    its mean."""
    X = np.array([[1.0], [2.0], [6.0], [0.0], [0.0], [3.0], [4.0], [4.0], [8.0], [-4.0]])
    assign, C = O.seal_window_blocks(X, 3)
    assert assign.tolist() == [0, 0, 0, 1, 1, 1, 2, 2, 2, 2]
    assert C[:, 0].tolist() == [3.0, 1.0, 3.0]
    idx = O.OracleIndex(d=1, n_sinks=2, window=10, clusters_per_window=3, refit_period=0,
                        block_routing=True)
    idx.append(np.concatenate([np.zeros((2, 1)), X, np.ones((3, 1))]))
    idx.seal()
    assert [c.members.tolist() for c in idx.clusters] == [[2, 3, 4], [5, 6, 7], [8, 9, 10, 11]]
    assert [(v.n_clusters, v.n_v) for v in idx.versions] == [(3, 12)]
    with pytest.raises(ValueError):
        O.OracleIndex(d=1, n_sinks=2, window=10, clusters_per_window=3, refit_period=10,
                      block_routing=True)
