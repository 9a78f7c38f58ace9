"""Helpers shared by the GPU parity tests: seeded inputs for both sides and
the matching rules.

Matching rules (exact unless a floating-point near tie makes several
results correct):
* index state (CSR offsets and members, bf16 representatives, versions) is
  compared exactly;
* a score agrees within 1e-3 * sum_h |w_h| ||q_h|| ||k|| of the float64
  value;
* candidate lists are equal, or differ only by clusters whose route scores
  are within that tolerance of each other (checked for validity);
* top-k sets are equal up to swaps whose scores are within tolerance of the
  k-th score;
* ids come out in (score desc, id asc) order: the library's own scores are
  sorted with ties broken by id, and the j-th id's float64 score lies
  within twice the tolerance of the oracle's j-th score.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import ai_oracle as O
from synth import workloads as S

REL_TOL = 1e-3


# ------------------------------------------------------------------ inputs --

def keys_inputs(wl: S.Workload, p0: int, p1: int, device="cuda"):
    """Keys [p0, p1): (device tensor for the library, scales or None,
    float64 values the oracle scores with)."""
    kf = S.keys_f64(wl, p0, p1)
    if wl.key_dtype == "fp32":
        k32 = kf.astype(np.float32)
        return torch.from_numpy(k32).to(device), None, k32.astype(np.float64)
    bits = S.to_bf16_bits(kf)
    kb = torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)
    vals = S.bf16_bits_to_f64(bits)
    if wl.key_dtype == "bf16":
        return kb, None, vals
    # fp8: the library quantises with its own kernel, the oracle with its own
    from ivf_top_key_b200 import quantize_fp8
    codes, scales = quantize_fp8(kb)
    ocodes, oscale = O.quantize_fp8_keys(vals.astype(np.float32))
    return codes, scales, ocodes * oscale.astype(np.float64)[:, None]


def query_inputs(wl: S.Workload, p0: int, p1: int, device="cuda"):
    q, w = S.queries_f64(wl, p0, p1)
    w32 = w.astype(np.float32)
    wd = torch.from_numpy(w32).to(device)
    if wl.q_dtype == "fp32":
        q32 = q.astype(np.float32)
        return torch.from_numpy(q32).to(device), wd, q32.astype(np.float64), w32.astype(np.float64)
    bits = S.to_bf16_bits(q)
    qd = torch.from_numpy(bits.view(np.int16)).to(device).view(torch.bfloat16)
    return qd, wd, S.bf16_bits_to_f64(bits), w32.astype(np.float64)


def make_pair(wl: S.Workload, encoder=None, async_refit=True, max_keys=None):
    from ivf_top_key_b200 import AttentionIndex
    gpu = AttentionIndex(
        d=wl.d, H=wl.H, key_dtype=wl.key_dtype, q_dtype=wl.q_dtype, n_sinks=wl.n_sinks,
        window=wl.window, clusters_per_window=wl.clusters_per_window,
        refit_period=wl.refit_period, refit_new_seeds=wl.refit_new_seeds,
        refit_seed_window=wl.refit_seed_window, seal_iters=wl.seal_iters,
        async_refit=async_refit, max_query_chunk=wl.T, max_budget=max(wl.budget, 64),
        max_k=wl.k, max_keys=max_keys or wl.L, seed=wl.seed, encoder_weights=encoder,
        block_routing=wl.block_routing)
    orc = O.OracleIndex(d=wl.d, n_sinks=wl.n_sinks, window=wl.window,
                        clusters_per_window=wl.clusters_per_window,
                        refit_period=wl.refit_period, refit_new_seeds=wl.refit_new_seeds,
                        refit_seed_window=wl.refit_seed_window, seal_iters=wl.seal_iters,
                        seed=wl.seed, encoder=encoder, block_routing=wl.block_routing)
    return gpu, orc


# ------------------------------------------------------------ tolerances --

def score_tol(q, w, keys):
    """1e-3 * sum_h |w_h| ||q_h|| ||k|| for each key row."""
    qn = np.linalg.norm(q, axis=1)
    return REL_TOL * (np.abs(w) * qn).sum() * np.linalg.norm(keys, axis=1)


# ------------------------------------------------------------- index state --

def check_index_equal(gpu, orc):
    ex = gpu.export_index()
    vn = [(v.n_clusters, v.n_v) for v in orc.versions]
    got_v = list(zip(ex["version_nc"].tolist(), ex["version_nv"].tolist()))
    assert got_v == vn, f"versions differ: {got_v[:5]} vs {vn[:5]}"
    nC = len(orc.clusters)
    assert ex["offsets"].shape[0] == nC + 1
    o_sizes = [c.members.size for c in orc.clusters]
    assert np.diff(ex["offsets"]).tolist() == o_sizes, "cluster sizes differ"
    o_mem = np.concatenate([c.members for c in orc.clusters]) if nC else np.zeros(0)
    bad = np.nonzero(ex["members"] != o_mem)[0]
    assert bad.size == 0, f"{bad.size} member slots differ, first at {bad[:5]}"
    reps = S.bf16_bits_to_f64(ex["reps_bf16"])
    orep = np.stack([c.rep for c in orc.clusters]) if nC else np.zeros((0, reps.shape[1]))
    nz = np.array(o_sizes) > 0
    diff = np.nonzero(np.any(reps[nz] != orep[nz], axis=1))[0]
    assert diff.size == 0, f"{diff.size} representatives differ"
    return ex


# ----------------------------------------------------------- query checks --

def check_sequence(t, ids, gpu_scores, exact, want_scores, tol_max):
    """The documented output order (score desc, id asc), position by position.

    ids / gpu_scores: the valid ids and the library's scores for them, in
    output order; exact: their float64 scores; want_scores: the oracle's
    top-k scores in its (score desc, id asc) order.  The library's own
    scores must be sorted with ties broken by id, and the j-th id's exact
    score must be within 2 * tol_max of the oracle's j-th score (a near-tie
    swap moves an id only among positions whose scores agree to that)."""
    gs = np.asarray(gpu_scores, dtype=np.float64)
    assert np.all(gs[1:] <= gs[:-1]), f"t={t}: scores not in descending order"
    tie = gs[1:] == gs[:-1]
    assert np.all(ids[1:][tie] > ids[:-1][tie]), f"t={t}: equal scores not in ascending id order"
    n = min(ids.size, want_scores.size)
    dev = np.abs(exact[:n] - want_scores[:n])
    assert np.all(dev <= 2 * tol_max + 1e-6), \
        f"t={t}: position {int(np.argmax(dev))} holds a score {dev.max():.3g} from the oracle's"


def check_queries(orc, t_list, q, w, gpu_ids, gpu_scores, gpu_cand, k, C, stats):
    """Compare route+refine results of the listed queries with the oracle:
    candidate lists, scores, the top-k set and its (score desc, id asc)
    order."""
    for i, t in enumerate(t_list):
        qi, wi = q[i], w[i]
        o_cand, rs, v = orc.candidates(t, qi, wi, C)
        g_cand = gpu_cand[i][gpu_cand[i] >= 0]
        g_ids = gpu_ids[i]
        valid = g_ids[g_ids >= 0]
        assert np.all(g_ids[valid.size:] == -1), f"t={t}: padding is not a -1 suffix"
        assert np.all(valid <= t), f"t={t}: selected a future key"
        assert len(set(valid.tolist())) == valid.size, f"t={t}: duplicate ids"
        # scores of the selected ids agree with float64
        exact = O.indexer_score(qi, wi, orc.keys[valid])
        tol = score_tol(qi, wi, orc.keys[valid])
        gs = gpu_scores[i][:valid.size]
        assert np.all(np.abs(gs - exact) <= tol + 1e-6), f"t={t}: score mismatch {np.max(np.abs(gs-exact)-tol)}"
        if np.array_equal(g_cand, o_cand):
            stats["cand_equal"] += 1
        else:
            stats["cand_near_tie"] += 1
            _check_candidate_validity(orc, t, qi, wi, g_cand, o_cand, rs, v, C)
        # top-k of the GPU's candidate set, with oracle scores
        cs = O.indexer_score(qi, wi, orc.keys[g_cand])
        want, want_sc = O.topk_ids(cs, g_cand, k)
        wv = want[want >= 0]
        assert valid.size == wv.size, f"t={t}: {valid.size} ids vs {wv.size}"
        tmax = float(score_tol(qi, wi, orc.keys[g_cand]).max()) if g_cand.size else 0.0
        check_sequence(t, valid, gs, exact, want_sc[:wv.size], tmax)
        if np.array_equal(valid, wv):
            stats["topk_equal"] += 1
        else:
            if set(valid.tolist()) != set(wv.tolist()):
                theta = want_sc[wv.size - 1]
                extra = np.setdiff1d(valid, wv)
                miss = np.setdiff1d(wv, valid)
                for s in np.concatenate([extra, miss]):
                    sc = O.indexer_score(qi, wi, orc.keys[[s]])[0]
                    tl = score_tol(qi, wi, orc.keys[[s]])[0]
                    assert abs(sc - theta) <= 2 * tl + 1e-6, f"t={t}: swap of key {s} not a near tie"
            stats["topk_near_tie"] += 1


def check_exhaustive(orc, t, q, w, got, got_sc, k):
    """Exhaustive selection of query t against the oracle's: the -1 padding,
    the set up to near-tie swaps at the k-th score, scores within tolerance
    and the (score desc, id asc) order."""
    want, want_sc = orc.exhaustive(q, w, t, k)
    vs = got >= 0
    assert np.array_equal(vs, np.arange(k) < min(k, t + 1)), f"t={t}: padding"
    g = got[vs]
    w_ = want[want >= 0]
    exact = O.indexer_score(q, w, orc.keys[g])
    tol = score_tol(q, w, orc.keys[g])
    assert np.all(np.abs(got_sc[vs] - exact) <= tol + 1e-6), f"t={t}: exhaustive score"
    tmax = float(score_tol(q, w, orc.keys[:t + 1]).max())
    check_sequence(t, g, got_sc[vs], exact, want_sc[:w_.size], tmax)
    if set(g.tolist()) != set(w_.tolist()):
        theta = want_sc[w_.size - 1]
        for s in np.setxor1d(g, w_):
            sc = O.indexer_score(q, w, orc.keys[[s]])[0]
            tl = score_tol(q, w, orc.keys[[s]])[0]
            assert abs(sc - theta) <= 2 * tl + 1e-6, f"t={t}: exhaustive swap {s}"
        return "exh_near_tie"
    return "exh_equal"


def _check_candidate_validity(orc, t, q, w, g_cand, o_cand, rs, v, C):
    S0 = orc.S
    n_fixed = min(S0, t + 1) + max(0, t + 1 - max(v.n_v, S0))
    assert np.array_equal(g_cand[:n_fixed], o_cand[:n_fixed]), f"t={t}: sinks/open differ"
    member_of = {}
    for c in range(v.n_clusters):
        for s in orc.clusters[c].members.tolist():
            member_of[s] = c
    order = []
    for s in g_cand[n_fixed:].tolist():
        c = member_of[s]
        if not order or order[-1] != c:
            assert c not in order, f"t={t}: cluster {c} split"
            order.append(c)
    reps = np.stack([orc.clusters[c].rep for c in range(v.n_clusters)])
    tol = score_tol(q, w, reps)
    for a, b in zip(order, order[1:]):
        assert rs[a] >= rs[b] - tol[a] - tol[b], f"t={t}: clusters {a},{b} out of order"
    if order:
        last = order[-1]
        sizes = np.array([orc.clusters[c].members.size for c in range(v.n_clusters)])
        for c in range(v.n_clusters):
            if c not in order and sizes[c] > 0:
                assert rs[c] <= rs[last] + tol[c] + tol[last], f"t={t}: cluster {c} skipped"
    assert g_cand.size == min(C, o_cand.size) or g_cand.size == o_cand.size
