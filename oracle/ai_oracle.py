"""CPU oracle for causal IVF top-k key selection (TEST INFRASTRUCTURE ONLY).

Only tests, the package's smoke check and the benchmark's CPU-baseline leg
may import this module.  The product path never calls it.

Plain, slow, float64 restatement of what the AttentionIndex method computes,
written from its description on the pages titled "AttentionIndex:
Accelerating Learned Sparse Attention with a Causal Inverted-File Index":

* explainer = paper-daily.com page, sections
  "它到底在解决什么问题？" (problem), "查询时怎么挑候选？" (query-time candidate
  fill), "索引怎么边算边建？" (insert / seal / refit / versions),
  "代表向量为什么要学？" (representatives and the learned correction, with the
  worked example box).
* review = kurate.org page, "Abstract" and "Impact Assessment: Core
  Contribution" (names size-capped k-means, Elkan/Hamerly bounds, DeepSets
  encoder, side-stream refits).

Precision: everything is float64 on the exact values the GPU consumes (bf16
bits, fp8 codes times their fp32 scale, fp32).  Two decisions are taken in
the precision the method fixes for its storage formats: representatives are
rounded to bf16 (round to nearest even) and fp8 key codes are chosen from
the float32 quotient key/scale.

Readings where the pages are silent (each also listed in the design notes):
sinks are the first S keys and are never clustered; query t sees keys
0..t; windows are [S + jW, S + (j+1)W); seal k-means uses strided init,
greedy global capacity assignment by (distance, key, cluster) and at most
`iters` iterations; refit is one brute-force Lloyd step from the previous
refit's centroids plus seeds drawn without replacement from recent keys by
a SplitMix64 counter generator; ties in every ranking go to the lower id;
an asynchronous refit becomes visible at the next append (or explicit
publish).

Parity pins: see tests/test_oracle_pins.py.  The encoder (learned
correction) is pinned by its zero-output case, its norm bound and closed
forms of each stage under hand-chosen weights; its architecture itself is
a reading of the explainer (the pages give no shapes).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

MASK64 = (1 << 64) - 1


# ---------------------------------------------------------------- formats --

def bf16_rne(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bfloat16 (ties to even).

    bfloat16 keeps 8 significant bits.  With x = m * 2**e, 0.5 <= |m| < 1,
    the rounded value is rint(m * 2**8) * 2**(e - 8) (np.rint rounds half to
    even).  Values are O(1) here; the bf16 subnormal range is not used.
    """
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    return np.ldexp(np.rint(m * 256.0), e - 8)


def e4m3_rne(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to FP8 E4M3 (OCP: bias 7, 3 mantissa bits,
    max finite 448, subnormals k * 2**-9), ties to even, saturating at +-448.

    Returns the rounded values as float64 (exactly representable)."""
    x = np.asarray(x32, dtype=np.float64)
    a = np.abs(x)
    out = np.zeros_like(a)
    nz = a > 0
    # exponent of the leading bit, clamped to the normal range [-6, 8]
    e = np.floor(np.log2(np.where(nz, a, 1.0)))
    # log2 can be off by one at exact powers of two: correct it
    e = np.where(np.ldexp(1.0, e.astype(np.int64)) > a, e - 1, e)
    e = np.where(np.ldexp(1.0, (e + 1).astype(np.int64)) <= a, e + 1, e)
    e = np.maximum(e, -6.0)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))  # spacing at that exponent
    r = np.rint(a / quantum) * quantum
    r = np.minimum(r, 448.0)
    out[nz] = r[nz]
    return np.sign(x) * out


def quantize_fp8_keys(keys_f32: np.ndarray):
    """Per-token scale = amax / 448 (float32), code = e4m3(key / scale).

    Returns (codes as float64 values, scales float32).  A zero row gets
    scale 1 and zero codes."""
    k32 = np.asarray(keys_f32, dtype=np.float32)
    amax = np.max(np.abs(k32), axis=1).astype(np.float32)
    scale = (amax / np.float32(448.0)).astype(np.float32)
    scale = np.where(amax > 0, scale, np.float32(1.0)).astype(np.float32)
    q32 = (k32 / scale[:, None]).astype(np.float32)
    return e4m3_rne(q32), scale


# ----------------------------------------------------------- score, top-k --

def indexer_score(q: np.ndarray, w: np.ndarray, keys: np.ndarray) -> np.ndarray:
    """DSA indexer score I(q, s) = sum_h w_h * ReLU(q_h . k_s).

    q [H, d], w [H], keys [n, d] -> [n].  (explainer, "代表向量为什么要学？":
    per-head inner products, ReLU, weighted sum; the same score ranks
    representatives and candidates.)"""
    dots = keys @ q.T                      # [n, H]
    return np.maximum(dots, 0.0) @ w        # [n]


def topk_ids(scores: np.ndarray, ids: np.ndarray, k: int):
    """The k largest scores, ordered by (score desc, id asc); pad with -1."""
    order = np.lexsort((ids, -scores))[:k]
    out_ids = np.full(k, -1, dtype=np.int64)
    out_sc = np.full(k, -np.inf)
    out_ids[:order.size] = ids[order]
    out_sc[:order.size] = scores[order]
    return out_ids, out_sc


def exhaustive_select(q: np.ndarray, w: np.ndarray, keys: np.ndarray, t: int, k: int):
    """Full DSA selection for the query at position t: score every key
    s <= t and keep the top k (explainer, "它到底在解决什么问题？")."""
    ids = np.arange(t + 1)
    return topk_ids(indexer_score(q, w, keys[:t + 1]), ids, k)


# ------------------------------------------------------------------ seal --

def seal_window(X: np.ndarray, m: int, cap: int, iters: int):
    """Size-capped k-means of one sealed window into m clusters.

    (explainer, "索引怎么边算边建？" item 2: every W open keys are grouped
    into m clusters and appended; review, "Core Contribution" item 1:
    size-capped k-means.)  The pages give no algorithm; this reading:
      init   c_j = X[floor((j + 1/2) W / m)]
      repeat at most `iters` times, stopping once the assignment repeats:
        D_ij = ||x_i - c_j||^2
        walk all (i, j) pairs by (D asc, i asc, j asc); give i to j if i is
        still free and j holds fewer than cap keys
        c_j = mean of its members (kept when empty)
    Returns (assign [W] int, centroids [m, d] float64).
    """
    W = X.shape[0]
    C = np.stack([X[((2 * j + 1) * W) // (2 * m)] for j in range(m)]).astype(np.float64)
    ii, jj = np.meshgrid(np.arange(W), np.arange(m), indexing="ij")
    ii = ii.ravel()
    jj = jj.ravel()
    prev = None
    assign = None
    for _ in range(iters):
        D = ((X[:, None, :] - C[None, :, :]) ** 2).sum(-1).ravel()
        order = np.lexsort((jj, ii, D))
        assign = np.full(W, -1, dtype=np.int64)
        count = np.zeros(m, dtype=np.int64)
        n_free = W
        for p in order:
            i, j = ii[p], jj[p]
            if assign[i] < 0 and count[j] < cap:
                assign[i] = j
                count[j] += 1
                n_free -= 1
                if n_free == 0:
                    break
        for j in range(m):
            mem = assign == j
            if mem.any():
                C[j] = X[mem].mean(axis=0)
        if prev is not None and np.array_equal(prev, assign):
            break
        prev = assign
    return assign, C


def seal_window_blocks(X: np.ndarray, m: int):
    """The contiguous-block baseline the explainer compares against
    ("它到底在解决什么问题？": HiSA groups keys by position into blocks, each
    scored through one representative).  Reading: block j of a window of W
    keys holds keys [floor(j W / m), floor((j + 1) W / m)), represented by
    their mean.  Returns (assign [W], centroids [m, d] float64)."""
    W = X.shape[0]
    starts = [(j * W) // m for j in range(m + 1)]
    assign = np.empty(W, dtype=np.int64)
    C = np.zeros((m, X.shape[1]))
    for j in range(m):
        assign[starts[j]:starts[j + 1]] = j
        if starts[j + 1] > starts[j]:
            C[j] = X[starts[j]:starts[j + 1]].mean(axis=0)
    return assign, C


# ----------------------------------------------------------------- refit --

def splitmix64(seed: int, ctr: int) -> int:
    """Counter-based SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): the
    output mix of state seed + (ctr + 1) * golden-gamma."""
    z = (seed + (ctr + 1) * 0x9E3779B97F4A7C15) & MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def refit_seed_ids(seed: int, refit_index: int, lo: int, hi: int, n_seed: int) -> np.ndarray:
    """n_seed distinct key ids drawn uniformly from [lo, hi), in draw order.

    Partial Fisher-Yates shuffle; draw i swaps slot i with slot
    i + splitmix64(seed, (refit_index << 32) | i) mod (n - i)."""
    n = hi - lo
    s = min(n_seed, n)
    perm = {}
    out = np.empty(s, dtype=np.int64)
    for i in range(s):
        r = splitmix64(seed, (refit_index << 32) | i)
        j = i + r % (n - i)
        vi = perm.get(i, i)
        vj = perm.get(j, j)
        perm[i], perm[j] = vj, vi
        out[i] = lo + vj
    return out


def refit_lloyd(X: np.ndarray, init_centroids: np.ndarray):
    """One warm-started assign + update pass over all clustered keys.

    (explainer, "索引怎么边算边建？" item 3 and the paragraph after it: start
    from the previous centres plus a few new ones from recent keys, one
    round of assignment and update.)  The Hamerly/Elkan bounds the pages
    name only skip distance computations whose outcome they already know,
    so the result is that of plain nearest-centre assignment, computed here
    by brute force.  Ties go to the lower centre id; an empty cluster keeps
    its centre.
    Returns (assign [n], centroids [K, d])."""
    K = init_centroids.shape[0]
    assign = np.empty(X.shape[0], dtype=np.int64)
    step = 4096
    for a in range(0, X.shape[0], step):
        xb = X[a:a + step]
        D = ((xb * xb).sum(1)[:, None] - 2.0 * (xb @ init_centroids.T)
             + (init_centroids * init_centroids).sum(1)[None, :])
        assign[a:a + step] = np.argmin(D, axis=1)   # first minimum = lower id
    C = init_centroids.copy()
    sums = np.zeros_like(C)
    np.add.at(sums, assign, X)
    cnt = np.bincount(assign, minlength=K)
    nz = cnt > 0
    C[nz] = sums[nz] / cnt[nz, None]
    return assign, C


# --------------------------------------------------------------- encoder --

def encoder_correction(members: np.ndarray, mu: np.ndarray, wts: dict) -> np.ndarray:
    """Bounded learned correction to a cluster mean (our reading).

    (explainer, "代表向量为什么要学？": a small shared network per layer reads
    the member mean, the log cluster size, and the mean and max of a learned
    per-key transform; its output is a bounded correction added to the mean,
    zero at initialisation.)  Reading:
      phi(k) = ReLU(A k + a)
      f = [mean phi ; max phi ; mu ; ln n]
      h = ReLU(B1 f + b1);  t = tanh(B2 h + b2)
      corr = t * min(1, 0.25 ||mu|| / ||t||)   (0 when t = 0)
    """
    A = wts["A"].astype(np.float64)
    phi = np.maximum(members @ A.T + wts["a"], 0.0)
    f = np.concatenate([phi.mean(0), phi.max(0), mu, [math.log(members.shape[0])]])
    h = np.maximum(wts["B1"].astype(np.float64) @ f + wts["b1"], 0.0)
    t = np.tanh(wts["B2"].astype(np.float64) @ h + wts["b2"])
    tn = float(np.sqrt((t * t).sum()))
    if tn == 0.0:
        return np.zeros_like(mu)
    bound = 0.25 * float(np.sqrt((mu * mu).sum()))
    return t * min(1.0, bound / tn)


# ----------------------------------------------------------------- index --

@dataclasses.dataclass
class Cluster:
    centroid: np.ndarray     # float64 [d]
    members: np.ndarray      # ascending key ids
    rep: np.ndarray          # bf16-rounded representative, as float64 [d]


@dataclasses.dataclass
class Version:
    n_clusters: int          # visible prefix of the cluster array
    n_v: int                 # watermark: keys [S, n_v) are clustered


class OracleIndex:
    """One (request, layer) causal IVF index, mirroring the library calls.

    State follows the explainer's "索引怎么边算边建？": appended keys (insert),
    sealed windows appended as clusters, refit results that replace the
    clustered prefix, and a version per seal / refit.  The cluster array is
    [clusters of the current refit base] ++ [clusters sealed after it]; each
    version is a prefix of it plus an open-window watermark.
    """

    def __init__(self, *, d, n_sinks, window, clusters_per_window, refit_period,
                 refit_new_seeds=0, refit_seed_window=0, seal_iters=10, seed=0,
                 encoder=None, cluster_cap=0, block_routing=False):
        self.d = d
        self.S = n_sinks
        self.W = window
        self.m = clusters_per_window
        self.cap = cluster_cap or -(-window // clusters_per_window)
        self.R = refit_period
        self.n_seed = refit_new_seeds or (refit_period * clusters_per_window // window if window else 0)
        self.seed_window = refit_seed_window or refit_period
        self.iters = seal_iters
        self.seed = seed
        self.encoder = encoder
        self.block_routing = block_routing
        if block_routing and (refit_period or encoder is not None):
            raise ValueError("block routing takes no refit and no encoder")
        self.keys = np.zeros((0, d))
        self.n_windows = 0
        self.clusters: list[Cluster] = []
        self.versions: list[Version] = []
        self.base_n_r = None               # watermark of the published base
        self.base_centroids = None         # most recent refit centroids
        self.pending = None                # (n_r, clusters, centroids)
        self.n_refits = 0
        self.refit_log = []                # (n_r, seed ids, assign) per refit

    # -- representatives
    def _make_cluster(self, centroid, members):
        if members.size and self.encoder is not None:
            corr = encoder_correction(self.keys[members], centroid, self.encoder)
        else:
            corr = 0.0
        return Cluster(centroid=centroid, members=members, rep=bf16_rne(centroid + corr))

    # -- insert (explainer, "索引怎么边算边建？" item 1)
    def append(self, keys_f64: np.ndarray):
        self.publish()
        self.keys = np.concatenate([self.keys, keys_f64], axis=0)

    # -- seal (item 2): every complete window, appended; refit every R tokens
    def seal(self):
        while self.keys.shape[0] >= self.S + (self.n_windows + 1) * self.W:
            lo = self.S + self.n_windows * self.W
            X = self.keys[lo:lo + self.W]
            if self.block_routing:
                assign, C = seal_window_blocks(X, self.m)
            else:
                assign, C = seal_window(X, self.m, self.cap, self.iters)
            for j in range(self.m):
                mem = lo + np.nonzero(assign == j)[0]
                self.clusters.append(self._make_cluster(C[j], mem))
            self.n_windows += 1
            self.versions.append(Version(len(self.clusters), lo + self.W))
            if self.R and (self.n_windows * self.W) % self.R == 0:
                self.refit()

    # -- refit (item 3)
    def refit(self):
        self.publish()
        n_r = self.S + self.n_windows * self.W
        if n_r <= self.S:
            return
        lo = max(self.S, n_r - self.seed_window)
        seeds = refit_seed_ids(self.seed, self.n_refits, lo, n_r, self.n_seed)
        init = self.keys[seeds]
        if self.base_centroids is not None:
            init = np.concatenate([self.base_centroids, init], axis=0)
        X = self.keys[self.S:n_r]
        assign, C = refit_lloyd(X, init)
        clusters = []
        for j in range(C.shape[0]):
            mem = self.S + np.nonzero(assign == j)[0]
            clusters.append(self._make_cluster(C[j], mem))
        self.refit_log.append((n_r, seeds, assign))
        self.n_refits += 1
        self.pending = (n_r, clusters, C)

    def publish(self):
        """Make a pending refit the new base (explainer: versions)."""
        if self.pending is None:
            return
        n_r, base, C = self.pending
        self.pending = None
        after = []
        newv = [Version(len(base), n_r)]
        # clusters sealed after n_r are kept, in seal order, after the base
        old_prev = 0
        for v in self.versions:
            if v.n_v > n_r:
                after.extend(self.clusters[old_prev:v.n_clusters])
                newv.append(Version(len(base) + len(after), v.n_v))
            old_prev = v.n_clusters
        self.clusters = base + after
        self.versions = newv
        self.base_n_r = n_r
        self.base_centroids = C

    # -- query side (explainer, "查询时怎么挑候选？" and the version paragraph)
    def version_for(self, t: int) -> Version:
        best = Version(0, self.S)
        for v in self.versions:
            if v.n_v <= t + 1:
                best = v
        return best

    def route_scores(self, q, w, n_clusters):
        if n_clusters == 0:
            return np.zeros(0)
        reps = np.stack([c.rep for c in self.clusters[:n_clusters]])
        return indexer_score(q, w, reps)

    def candidates(self, t, q, w, C):
        v = self.version_for(t)
        cand = list(range(min(self.S, t + 1)))
        cand += list(range(max(v.n_v, self.S), t + 1))
        sc = self.route_scores(q, w, v.n_clusters)
        order = np.lexsort((np.arange(v.n_clusters), -sc))
        for c in order:
            if len(cand) >= C:
                break
            cand.extend(self.clusters[c].members.tolist())
        return np.asarray(cand[:C], dtype=np.int64), sc, v

    def route_refine(self, q, w, t, k, C):
        cand, _, _ = self.candidates(t, q, w, C)
        return topk_ids(indexer_score(q, w, self.keys[cand]), cand, k)

    def exhaustive(self, q, w, t, k):
        return exhaustive_select(q, w, self.keys, t, k)


def recall(selected: np.ndarray, reference: np.ndarray) -> float:
    """Micro-averaged recall: sum_t |sel_t & ref_t| / sum_t |ref_t| over
    valid (>= 0) ids (explainer, "它到底在解决什么问题？" defines recall as the
    share of the exhaustive top-k recovered)."""
    hit = 0
    tot = 0
    for s, r in zip(selected, reference):
        r = r[r >= 0]
        hit += np.intersect1d(s[s >= 0], r).size
        tot += r.size
    return hit / max(tot, 1)
