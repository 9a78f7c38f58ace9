"""Full-size GPU parity, in the launch configuration the benchmark times
(8192-query chunks, refit on the side stream).

* 128K-key bf16 (32 heads) and 256K-key fp8 (64 heads) prefills: the float64
  oracle runs the whole prefill beside the library (it finishes in seconds
  to a minute at these sizes); the index state is compared exactly after
  every chunk, route+refine on sampled queries of every chunk, exhaustive
  selection on sampled queries of the last chunk.
* 1M-key bf16 prefill: too large for the oracle's brute-force refits, so
  each step is checked where it can be computed one output at a time, on
  the library's own exported state: the last refit's assignment of sampled
  keys (oracle nearest-centre pass from the previous base centres plus the
  oracle's seed draw), the update (centres are member means, reps their
  bf16 rounding), the windows sealed after that refit (oracle seal, exact),
  route+refine and exhaustive selection of sampled queries of the last
  chunk (oracle candidate fill and top-k over the exported clusters).
"""
import collections

import numpy as np
import pytest
import torch

from oracle import ai_oracle as O
from synth import workloads as S
from tests import parity as P

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

if not torch.cuda.is_available():  # pragma: no cover
    pytest.skip("needs a GPU", allow_module_level=True)

from tests.test_gpu_parity import _run_prefill  # noqa: E402


def test_glm_bf16_L128k_full_prefill():
    wl = S.WORKLOADS["glm_bf16_L128k"]
    st = _run_prefill(wl, sample=6, check_exhaustive={wl.n_chunks - 1})
    n = st["cand_equal"] + st["cand_near_tie"]
    assert st["cand_near_tie"] <= 0.05 * n, st


def test_v4flash_fp8_L256k_full_prefill():
    wl = S.WORKLOADS["v4flash_fp8_L256k"]
    st = _run_prefill(wl, sample=3, check_exhaustive={wl.n_chunks - 1})
    n = st["cand_equal"] + st["cand_near_tie"]
    assert st["cand_near_tie"] <= 0.05 * n, st


def _oracle_view(ex, keys, wl):
    """An oracle index holding the library's exported clusters and versions
    (the candidate fill and top-k then run with the oracle's arithmetic)."""
    orc = O.OracleIndex(d=wl.d, n_sinks=wl.n_sinks, window=wl.window,
                        clusters_per_window=wl.clusters_per_window, refit_period=wl.refit_period,
                        seed=wl.seed)
    orc.keys = keys
    off = ex["offsets"]
    reps = S.bf16_bits_to_f64(ex["reps_bf16"])
    orc.clusters = [O.Cluster(centroid=ex["centroids"][c], members=ex["members"][off[c]:off[c + 1]],
                              rep=reps[c]) for c in range(off.size - 1)]
    orc.versions = [O.Version(int(a), int(b)) for a, b in zip(ex["version_nc"], ex["version_nv"])]
    return orc


def _bf16_rounding_agrees(got_bits, centroids):
    """reps == bf16(centroid), allowing a different rounding only where the
    centroid sits within 1e-12 (relative) of a bf16 rounding midpoint."""
    want = O.bf16_rne(centroids)
    got = S.bf16_bits_to_f64(got_bits)
    bad = got != want
    if not bad.any():
        return True
    c = centroids[bad]
    mid = 0.5 * (got[bad] + want[bad])
    return bool(np.all(np.abs(c - mid) <= 1e-12 * np.abs(c)))


def test_glm_bf16_L1m_sampled_steps():
    wl = S.WORKLOADS["glm_bf16_L1m"]
    gpu, _ = P.make_pair(wl)
    rng = np.random.default_rng(99)
    keys = np.empty((wl.L, wl.d))
    prev_ex = None
    last = None  # (export before the refit, n_refits before it)
    for c in range(wl.n_chunks):
        p0, p1 = c * wl.T, (c + 1) * wl.T
        kd, ks, kv = P.keys_inputs(wl, p0, p1)
        keys[p0:p1] = kv
        before = gpu.stats()["n_refits"]
        gpu.append_keys(kd, ks)
        gpu.seal()
        if gpu.stats()["n_refits"] > before:
            last = (prev_ex, before)
        if c >= wl.n_chunks - 24:
            # keep the published state of the chunks near the end: the last
            # refit's inputs are read from the export taken just before it
            gpu.publish()
            gpu.sync()
            prev_ex = gpu.export_index()
    gpu.publish()
    gpu.sync()
    ex = gpu.export_index()
    assert last is not None and last[0] is not None, "no refit among the last chunks"
    ex_prev, r = last
    Sk, W, m = wl.n_sinks, wl.window, wl.clusters_per_window
    off = ex["offsets"]
    n_base, n_r = int(ex["version_nc"][0]), int(ex["version_nv"][0])

    # partition: every clustered key in exactly one cluster
    mem = ex["members"]
    assert mem.size == int(ex["version_nv"][-1]) - Sk
    assert np.array_equal(np.sort(mem), np.arange(Sk, Sk + mem.size))

    # the last refit: assignment of sampled keys against its initial centres
    K_prev = int(ex_prev["version_nc"][0]) if ex_prev["version_nc"].size else 0
    prev_n_r = int(ex_prev["version_nv"][0]) if ex_prev["version_nv"].size else Sk
    assert prev_n_r < n_r
    n_seed = wl.refit_new_seeds or wl.refit_period * m // W
    seed_window = wl.refit_seed_window or wl.refit_period
    seeds = O.refit_seed_ids(wl.seed, r, max(Sk, n_r - seed_window), n_r, n_seed)
    init = np.concatenate([ex_prev["centroids"][:K_prev], keys[seeds]], axis=0)
    assert n_base == init.shape[0]
    owner = np.empty(wl.L, dtype=np.int64)
    for cl in range(n_base):
        owner[mem[off[cl]:off[cl + 1]]] = cl
    xs = np.sort(rng.choice(np.arange(Sk, n_r), size=3000, replace=False))
    want, _ = O.refit_lloyd(keys[xs], init)
    got = owner[xs]
    diff = np.nonzero(want != got)[0]
    for i in diff:  # only float64 near ties may differ
        x = keys[xs[i]]
        da = ((x - init[want[i]]) ** 2).sum()
        db = ((x - init[got[i]]) ** 2).sum()
        assert abs(da - db) <= 1e-9 * (x @ x + init[got[i]] @ init[got[i]]), (xs[i], want[i], got[i])
    # update: base centres are the member means (an empty cluster keeps its
    # initial centre); reps are their bf16 rounding
    cents = ex["centroids"]
    sizes = np.diff(off)
    for cl in range(n_base):
        want_c = keys[mem[off[cl]:off[cl + 1]]].mean(0) if sizes[cl] else init[cl]
        assert np.allclose(cents[cl], want_c, rtol=1e-12, atol=1e-12), cl
    assert _bf16_rounding_agrees(ex["reps_bf16"], cents)

    # windows sealed after the last refit: exact against the oracle's seal
    cap = -(-W // m)
    for j, v in enumerate(ex["version_nv"][1:].tolist()):
        lo = v - W
        assign, C = O.seal_window(keys[lo:v], m, cap, wl.seal_iters)
        for jj in range(m):
            cl = n_base + j * m + jj
            assert np.array_equal(mem[off[cl]:off[cl + 1]], lo + np.nonzero(assign == jj)[0]), (v, jj)
            assert np.array_equal(S.bf16_bits_to_f64(ex["reps_bf16"][cl]), O.bf16_rne(C[jj])), (v, jj)

    # route+refine and exhaustive selection of sampled queries, last chunk
    orc = _oracle_view(ex, keys, wl)
    p0 = wl.L - wl.T
    qd, wd, qv, wv = P.query_inputs(wl, p0, wl.L)
    out = torch.full((wl.T, wl.k), -7, dtype=torch.int32, device="cuda")
    osc = torch.zeros((wl.T, wl.k), dtype=torch.float32, device="cuda")
    gpu.route_refine(qd, wd, p0, wl.k, wl.budget, out=out, out_scores=osc)
    cand, _ = gpu.debug_candidates(qd, wd, p0, wl.budget, with_scores=False)
    eo = torch.full((wl.T, wl.k), -7, dtype=torch.int32, device="cuda")
    es = torch.zeros((wl.T, wl.k), dtype=torch.float32, device="cuda")
    gpu.select_exhaustive(qd, wd, p0, wl.k, out=eo, out_scores=es)
    gpu.sync()
    idx = np.unique(np.concatenate([[0, wl.T - 1], rng.choice(wl.T, size=8, replace=False)]))
    stats = collections.Counter()
    P.check_queries(orc, (p0 + idx).tolist(), qv[idx], wv[idx], out.cpu().numpy()[idx],
                    osc.cpu().numpy()[idx], cand.cpu().numpy()[idx], wl.k, wl.budget, stats)
    eo, es = eo.cpu().numpy(), es.cpu().numpy()
    for i in idx[:4]:
        P.check_exhaustive(orc, p0 + i, qv[i], wv[i], eo[i], es[i], wl.k)
    gpu.close()
