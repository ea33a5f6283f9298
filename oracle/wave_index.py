"""Oracle for the wave-index path: a plain, slow, fp64 CPU restatement.

TEST INFRASTRUCTURE ONLY.  Nothing in the product imports, links or runs this
module; only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg do.  It shares no code with the CUDA path.

Sources (web pages about RetroInfer, arXiv:2505.02922), cited by title and
section:

* [P1] "微软新突破：RetroInfer如何让AI模型处理百万级文本不再'卡顿'？"
  (techwalker.com), sections 三 (wave index / wave buffer) and 四.
* [P2] "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn),
  §2.1 "Wave索引", §2.2 "Wave缓冲", §3.1, §3.3 "注意力计算的工程优化".
* [P3] "RetroInfer: A Vector-Storage Approach for Scalable Long-Context LLM
  Inference" (chatpaper.ai), abstract.
* [P4] "RetroInfer: A Vector Storage Engine for Scalable Long-Context LLM
  Inference" (gist.science), "Technische Samenvatting" §2A.

What the pages fix, in short: three zones per head (steady = first 4 and last
64 tokens, exact; retrieval = clusters picked by the index, about 1.8 % of
tokens, exact; estimation = next-ranked clusters, about 23 % of tokens,
approximated from each cluster's centroid and size) [P2 §2.1, §3.3; P3;
P4 §2A]; the index is k-means run separately on 8K-token segments, giving
centroids and per-cluster value sums [P2 §2.1 pseudocode]; partial results are
merged [P2 §3.3].  Readings where the pages are silent or garbled (all listed
in the design notes): steady tokens are not indexed; the budgets are cluster
counts round(0.018 C) and round(0.23 C); clusters outside both zones are
dropped; one selection per KV head scored by the sum of its query heads'
scores; 512 clusters per 8K segment (the garbled "centroids=16" read as 16
tokens per centroid); Lloyd's algorithm with given seeds, empty clusters
keeping their centroid, a fixed iteration count; ties go to the lower index;
centroids stored in bf16, value sums in fp32; softmax scale 1/sqrt(d).

All arithmetic is fp64 on bf16 inputs widened exactly.  Parity status of each
function is stated in its docstring; the only unpinned part is the pages'
"accuracy bound" of the estimation, which the pages never state and which is
therefore not computed here (parity unpinned).
"""
from __future__ import annotations

import math

import numpy as np

# [P2 §2.1 item 1]: the first 4 prompt tokens and the most recent 64 tokens.
STEADY_INITIAL = 4
STEADY_RECENT = 64
# [P2 §2.1 item 2]: k-means per 8K-token segment.
SEGMENT_TOKENS = 8192
# Reading of the garbled "centroids=16" in [P2 §2.1]: 16 tokens per centroid,
# i.e. 512 clusters per full 8K segment.
CLUSTERS_PER_SEGMENT = 512
# [P2 §2.1 items 2-3]: retrieval about 1.8 %, estimation about 23 %.
RETRIEVAL_FRACTION = 0.018
ESTIMATION_FRACTION = 0.23
# Lloyd iterations of the workloads (fixed count, no early stop).
DEFAULT_ITERS = 10


# --------------------------------------------------------------------------
# number formats
# --------------------------------------------------------------------------
def bf16_round(x) -> np.ndarray:
    """Round to the nearest bf16 value (8 significant bits, binary32 exponent
    range), ties to even, returned as fp64.  One rounding straight from the
    fp64 value: x = m * 2^e with m in [0.5, 1); keep round(m * 2^8) * 2^(e-8).
    Below the normal range the quantum is fixed at 2^-133.  Pinned against
    torch's bf16 conversion of fp32 inputs."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    out = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    tiny = np.abs(x) < 2.0 ** -126
    out = np.where(tiny, np.rint(x * 2.0 ** 133) * 2.0 ** -133, out)
    return np.where(np.isfinite(x), out, x)


# --------------------------------------------------------------------------
# zones and segments  [P2 §2.1; P1 三; P4 §2A]
# --------------------------------------------------------------------------
def steady_positions(N: int, s0: int = STEADY_INITIAL, s1: int = STEADY_RECENT) -> np.ndarray:
    """Token positions of the steady zone, in position order.

    [P2 §2.1 item 1]: the first 4 and the most recent 64 tokens.  With
    N <= 68 every token is steady."""
    if N <= s0 + s1:
        return np.arange(N, dtype=np.int64)
    return np.concatenate([np.arange(s0), np.arange(N - s1, N)]).astype(np.int64)


def middle_range(N: int, s0: int = STEADY_INITIAL, s1: int = STEADY_RECENT) -> tuple[int, int]:
    """(first position, count M) of the indexed middle tokens [4, N-64).

    Reading: the steady tokens are not indexed, so no token is counted twice."""
    M = max(0, N - s0 - s1)
    return (s0 if M > 0 else 0), M


def segments(M: int, seg_len: int = SEGMENT_TOKENS,
             clusters_per_seg: int = CLUSTERS_PER_SEGMENT) -> list[tuple[int, int, int]]:
    """Split M middle tokens into contiguous segments [P2 §2.1 pseudocode].

    Returns (start within the middle, length L_s, clusters K_s) per segment;
    the last segment may be short and has K_s = min(clusters, L_s)."""
    out = []
    start = 0
    while start < M:
        L = min(seg_len, M - start)
        out.append((start, L, min(clusters_per_seg, L)))
        start += L
    return out


def default_budgets(C: int) -> tuple[int, int]:
    """Cluster budgets (k_r, k_e) = round half up of 1.8 % and 23 % of C
    [P2 §2.1 items 2-3], read as cluster counts."""
    def rhu(x: float) -> int:
        return int(math.floor(x + 0.5))
    return rhu(RETRIEVAL_FRACTION * C), rhu(ESTIMATION_FRACTION * C)


def strided_init(L: int, K: int) -> np.ndarray:
    """Default seeding when none is given: positions floor(j * L / K)."""
    return (np.arange(K, dtype=np.int64) * L) // K


# --------------------------------------------------------------------------
# segmented clustering  [P2 §2.1 pseudocode; P3 abstract; P4 §2A]
# --------------------------------------------------------------------------
def assign(X: np.ndarray, mu: np.ndarray) -> np.ndarray:
    """Label of each row: the index of its nearest centroid in squared
    Euclidean distance, lowest index on ties.

    argmin_j ||x - mu_j||^2 = argmin_j (||mu_j||^2 - 2 x.mu_j): ||x||^2 does
    not depend on j.  The second form is used (one fp64 matmul); it is pinned
    against the direct difference form in the tests."""
    crit = (mu * mu).sum(axis=1)[None, :] - 2.0 * (X @ mu.T)
    return np.argmin(crit, axis=1).astype(np.int64)


def update(X: np.ndarray, labels: np.ndarray, mu_prev: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """New centroids = mean of each cluster's members; an empty cluster keeps
    its previous centroid.  Returns (mu, counts)."""
    K = mu_prev.shape[0]
    counts = np.bincount(labels, minlength=K).astype(np.int64)
    sums = np.zeros_like(mu_prev)
    np.add.at(sums, labels, X)
    mu = mu_prev.copy()
    nz = counts > 0
    mu[nz] = sums[nz] / counts[nz][:, None]
    return mu, counts


def objective(X: np.ndarray, labels: np.ndarray, mu: np.ndarray) -> float:
    """Sum over rows of ||x_i - mu_{label_i}||^2 (direct difference form)."""
    diff = X - mu[labels]
    return float((diff * diff).sum())


def kmeans(X: np.ndarray, init_pos, iters: int) -> dict:
    """Lloyd's k-means on one segment [P2 §2.1 pseudocode `kmeans(seg, k)`].

    mu^0 = X[init_pos]; for t = 1..T: labels^t = assign(X, mu^{t-1}),
    mu^t = update(X, labels^t, mu^{t-1}).  The result is (labels^T, mu^T), so
    every non-empty centroid is exactly the mean of its final members.  With
    T = 0 the labels are the assignment to the seeds and mu stays the seeds.
    `history` holds the objective of (labels^t, mu^t) after every iteration.
    """
    X = np.asarray(X, dtype=np.float64)
    mu = X[np.asarray(init_pos, dtype=np.int64)].copy()
    hist = []
    if iters == 0:
        labels = assign(X, mu)
        counts = np.bincount(labels, minlength=mu.shape[0])
        return dict(labels=labels, mu=mu, counts=counts, history=hist)
    for _ in range(iters):
        labels = assign(X, mu)
        mu, counts = update(X, labels, mu)
        hist.append(objective(X, labels, mu))
    return dict(labels=labels, mu=mu, counts=counts, history=hist)


def finalise(Kh: np.ndarray, Vh: np.ndarray, N: int, seg_labels: list[np.ndarray],
             seg_mu: list[np.ndarray], seg_len: int = SEGMENT_TOKENS,
             clusters_per_seg: int = CLUSTERS_PER_SEGMENT, s0: int = STEADY_INITIAL,
             s1: int = STEADY_RECENT) -> dict:
    """Index of one (sequence, KV head) from per-segment labels and centroids.

    * cluster-contiguous layout [P2 §3.1: the KV vectors of one cluster are
      stored contiguously]: clusters in global id order (segment-major), the
      members of one cluster in position order (a stable permutation);
    * per-cluster size n_c, offsets (row of the cluster's first token),
      value sum Vsum_c [P2 §2.1 `compute_cluster_sums`];
    * centroid stored as bf16 (round to nearest even) of mu;
    * steady buffer: the steady tokens' K and V in position order [P1 三: a
      small buffer holds the steady zone].

    Kh, Vh: fp64 [N][d] (exact widenings of the bf16 inputs).  Positions in
    `perm` are absolute token positions."""
    d = Kh.shape[1]
    m0, M = middle_range(N, s0, s1)
    segs = segments(M, seg_len, clusters_per_seg)
    C = sum(s[2] for s in segs)
    perm = np.empty(M, dtype=np.int64)
    counts = np.zeros(C, dtype=np.int64)
    offsets = np.zeros(C + 1, dtype=np.int64)
    centroid = np.zeros((C, d))
    vsum = np.zeros((C, d))
    mu_all = np.zeros((C, d))
    cbase = 0
    for (start, L, Ks), lab, mu in zip(segs, seg_labels, seg_mu):
        lab = np.asarray(lab, dtype=np.int64)
        order = np.argsort(lab, kind="stable")           # by cluster, then position
        perm[start:start + L] = m0 + start + order
        n = np.bincount(lab, minlength=Ks)
        counts[cbase:cbase + Ks] = n
        offsets[cbase:cbase + Ks] = start + np.concatenate([[0], np.cumsum(n)[:-1]])
        pos = m0 + start + np.arange(L)
        np.add.at(vsum[cbase:cbase + Ks], lab, Vh[pos])
        centroid[cbase:cbase + Ks] = bf16_round(mu)
        mu_all[cbase:cbase + Ks] = mu
        cbase += Ks
    offsets[C] = M
    sp = steady_positions(N, s0, s1)
    return dict(N=N, C=C, perm=perm, counts=counts, offsets=offsets,
                centroid=centroid, vsum=vsum, mu=mu_all,
                Kp=Kh[perm], Vp=Vh[perm], Ks=Kh[sp], Vs=Vh[sp])


def build_index_head(Kh, Vh, init_pos=None, iters: int = DEFAULT_ITERS,
                     seg_len: int = SEGMENT_TOKENS, clusters_per_seg: int = CLUSTERS_PER_SEGMENT,
                     s0: int = STEADY_INITIAL, s1: int = STEADY_RECENT) -> dict:
    """Segmented clustering of one (sequence, KV head) [P2 §2.1 pseudocode]:
    k-means on every segment independently, then `finalise`.

    init_pos: positions within each segment, concatenated over segments
    (length C), or None for strided seeding.  Adds per-segment labels and
    objective (of the final labels against the final fp64 centroids)."""
    Kh = np.asarray(Kh, dtype=np.float64)
    Vh = np.asarray(Vh, dtype=np.float64)
    N = Kh.shape[0]
    m0, M = middle_range(N, s0, s1)
    labs, mus, objs, hists = [], [], [], []
    cbase = 0
    for start, L, Ks in segments(M, seg_len, clusters_per_seg):
        X = Kh[m0 + start:m0 + start + L]
        ip = strided_init(L, Ks) if init_pos is None else np.asarray(init_pos[cbase:cbase + Ks])
        res = kmeans(X, ip, iters)
        labs.append(res["labels"])
        mus.append(res["mu"])
        objs.append(objective(X, res["labels"], res["mu"]))
        hists.append(res["history"])
        cbase += Ks
    idx = finalise(Kh, Vh, N, labs, mus, seg_len, clusters_per_seg, s0, s1)
    idx["labels"] = labs
    idx["objective"] = np.array(objs)
    idx["history"] = hists
    return idx


def index_from_labels(Kh, Vh, labels_middle: np.ndarray, seg_len: int = SEGMENT_TOKENS,
                      clusters_per_seg: int = CLUSTERS_PER_SEGMENT, s0: int = STEADY_INITIAL,
                      s1: int = STEADY_RECENT) -> dict:
    """Index of one head from given labels of the middle tokens (cluster id
    within the segment), centroids = member means (0 for empty clusters).

    Used to form large valid indexes without running k-means (the labels come
    from the input generator's planted components)."""
    Kh = np.asarray(Kh, dtype=np.float64)
    Vh = np.asarray(Vh, dtype=np.float64)
    N = Kh.shape[0]
    m0, M = middle_range(N, s0, s1)
    labs, mus = [], []
    for start, L, Ks in segments(M, seg_len, clusters_per_seg):
        lab = np.asarray(labels_middle[start:start + L], dtype=np.int64)
        X = Kh[m0 + start:m0 + start + L]
        mu, _ = update(X, lab, np.zeros((Ks, Kh.shape[1])))
        labs.append(lab)
        mus.append(mu)
    idx = finalise(Kh, Vh, N, labs, mus, seg_len, clusters_per_seg, s0, s1)
    idx["labels"] = labs
    return idx


# --------------------------------------------------------------------------
# decode: tripartite attention  [P2 §2.1, §2.2 step 1, §3.3; P4 §2A]
# --------------------------------------------------------------------------
def centroid_scores(q_group: np.ndarray, centroid: np.ndarray) -> np.ndarray:
    """s[g, c] = q_g . centroid_c / sqrt(d) for the G query heads of one KV
    head (querying the wave index for cluster ids, [P2 §2.2 step 1])."""
    d = q_group.shape[1]
    return (q_group @ centroid.T) / math.sqrt(d)


def select_clusters(r: np.ndarray, k_r: int, k_e: int) -> tuple[np.ndarray, np.ndarray]:
    """Rank clusters by selection key r (descending, lower id first on ties);
    the first k_r form the retrieval zone, the next k_e the estimation zone
    [P2 §2.1 items 2-3].  Both returned sorted by id."""
    C = r.shape[0]
    order = np.lexsort((np.arange(C), -r))       # primary -r, secondary id
    k_r = min(k_r, C)
    k_e = min(k_e, C - k_r)
    return np.sort(order[:k_r]), np.sort(order[k_r:k_r + k_e])


def tripartite_attention(q_group: np.ndarray, idx: dict, k_r: int, k_e: int) -> dict:
    """Decode attention of the G query heads of one KV head.

    Exact softmax terms over the steady tokens and the tokens of the
    retrieval clusters; for every estimation cluster c and query head h, c
    adds n_c * exp(s_hc) to the denominator and exp(s_hc) * Vsum_c to the
    numerator (centroid and size stand for the cluster, [P2 §3.3 item 1;
    P4 §2A]); tokens of other clusters are dropped.  Selection is shared by
    the G query heads with key r_c = sum_h s_hc (r_c = -inf for empty
    clusters).  Computed with one global max shift; lse = log of the
    denominator (natural log, unshifted)."""
    q = np.asarray(q_group, dtype=np.float64)
    G, d = q.shape
    scale = 1.0 / math.sqrt(d)
    C = idx["C"]
    if C > 0:
        s = centroid_scores(q, idx["centroid"])
        r = s.sum(axis=0)
        r = np.where(idx["counts"] > 0, r, -np.inf)
        R, E = select_clusters(r, k_r, k_e)
    else:
        s = np.zeros((G, 0))
        R = E = np.zeros(0, dtype=np.int64)
    rows = [np.arange(idx["offsets"][c], idx["offsets"][c] + idx["counts"][c]) for c in R]
    rows = np.concatenate(rows).astype(np.int64) if rows else np.zeros(0, dtype=np.int64)
    Kx = np.concatenate([idx["Ks"], idx["Kp"][rows]], axis=0)
    Vx = np.concatenate([idx["Vs"], idx["Vp"][rows]], axis=0)
    x = (q @ Kx.T) * scale                                   # [G][T_exact]
    nE = idx["counts"][E].astype(np.float64)
    sE = s[:, E]                                             # [G][k_e]
    live = nE > 0
    m = np.full(G, -np.inf)
    if x.shape[1]:
        m = np.maximum(m, x.max(axis=1))
    if live.any():
        m = np.maximum(m, sE[:, live].max(axis=1))
    px = np.exp(x - m[:, None])
    pe = np.where(live[None, :], np.exp(sE - m[:, None]), 0.0)
    num = px @ Vx + pe @ idx["vsum"][E]
    den = px.sum(axis=1) + pe @ nE
    out = num / den[:, None]
    lse = m + np.log(den)
    return dict(out=out, lse=lse, R=R, E=E, scores=s,
                exact_tokens=int(x.shape[1]), estimated_tokens=int(nE.sum()))


def decode(q: np.ndarray, index: list[list[dict]], k_r: int, k_e: int) -> dict:
    """Batched decode: q [B][H_kv*G][d]; index[b][h] per (sequence, KV head).
    Query head h_q uses KV head h_q // G."""
    q = np.asarray(q, dtype=np.float64)
    B, Hq, d = q.shape
    H = len(index[0])
    G = Hq // H
    out = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    R, E = [], []
    for b in range(B):
        Rb, Eb = [], []
        for h in range(H):
            res = tripartite_attention(q[b, h * G:(h + 1) * G], index[b][h], k_r, k_e)
            out[b, h * G:(h + 1) * G] = res["out"]
            lse[b, h * G:(h + 1) * G] = res["lse"]
            Rb.append(res["R"])
            Eb.append(res["E"])
        R.append(Rb)
        E.append(Eb)
    return dict(out=out, lse=lse, R=R, E=E)


# --------------------------------------------------------------------------
# LRU block cache (wave buffer)  [P2 §2.2; P4 §2B]
# --------------------------------------------------------------------------
class LRUClusterCache:
    """Reference model of the GPU block cache's bookkeeping: a mapping table
    cluster -> blocks and an LRU order over clusters [P2 §2.2 "同步访问路径" /
    "异步更新路径"; P2 §3.1: the cache is made of fixed 2 KB physical blocks,
    8 rows of 128 bf16 values].

    Capacity is counted in blocks; a cluster occupies `blocks(c)` of them
    (ceil(rows / 8) in the library; 1 when no sizes are given, so capacity is
    then counted in clusters).  `access(ids)` looks every requested cluster up
    (hit or miss), then admits the misses in request order, evicting least
    recently used clusters that are not requested in this same step until the
    miss fits; a miss that cannot fit even after every such eviction (larger
    than the free blocks plus those of the evictable residents) is served
    without being cached and evicts nothing.  All requested resident clusters
    become most recent, in request order.  A
    cluster of zero blocks holds no rows: it counts as a hit and is not
    tracked.  Returns (hits, misses) lists."""

    def __init__(self, capacity: int, blocks=None):
        self.capacity = capacity
        self.blocks = blocks if blocks is not None else (lambda c: 1)
        self.slot_of: dict[int, list[int]] = {}
        self.order: list[int] = []          # least recent first
        self.free = list(range(capacity))[::-1]

    def access(self, ids) -> tuple[list[int], list[int]]:
        ids = [int(i) for i in ids]
        hits = [i for i in ids if i in self.slot_of or self.blocks(i) == 0]
        misses = [i for i in ids if i not in self.slot_of and self.blocks(i) > 0]
        req = set(ids)
        for i in misses:
            need = self.blocks(i)
            evictable = sum(len(self.slot_of[v]) for v in self.order if v not in req)
            if len(self.free) + evictable < need:
                continue                    # cannot fit: served uncached, nothing evicted
            while len(self.free) < need:
                victim = next(v for v in self.order if v not in req)
                self.order.remove(victim)
                self.free.extend(self.slot_of.pop(victim))
            self.slot_of[i] = [self.free.pop() for _ in range(need)]
            self.order.append(i)
        for i in ids:
            if i in self.slot_of:
                self.order.remove(i)
                self.order.append(i)
        return hits, misses


# --------------------------------------------------------------------------
# index maintenance during decode  [P2 §2.1 item 1 and pseudocode; reading]
# --------------------------------------------------------------------------
def open_slots(seg_len: int, k_last: int) -> int:
    """Member slots of one open cluster when the last closed segment has
    k_last clusters: ceil(2 * seg_len / k_last) (reading: twice the mean
    occupancy, so the open segment always has room for seg_len tokens)."""
    return -(-2 * seg_len // k_last)


class GrowingIndex:
    """The wave index of one (sequence, KV head) kept up to date while the
    sequence grows by one token per decode step.

    The pages fix the zones (the steady zone holds the first 4 and the most
    recent 64 tokens, [P2 §2.1 item 1]) and that the index is k-means over
    8K-token segments [P2 §2.1 pseudocode]; they are silent on what happens
    to a token that leaves the recent window.  Reading (the plainest that
    keeps every token in exactly one zone and the index segmented):

    * appending token N moves token N - s1 out of the recent window into the
      *open segment*;
    * the open segment has K open clusters (K = min(clusters, seg_len)); the
      moving token joins open cluster j, where j is its nearest centroid
      (squared Euclidean distance to the stored bf16 centroids, lower id on
      ties) among the K_last clusters of the last closed segment, counting
      only clusters with a free slot (each open cluster has
      ceil(2 seg_len / K_last) slots); n_j and Vsum_j grow by the token; open
      cluster j is scored with
      the centroid of cluster j of the last closed segment (the open clusters
      beyond K_last stay empty);
    * when the open segment holds seg_len tokens it is closed: k-means over
      its tokens in position order (seeds floor(j L / K), the build's
      iteration count) makes it a closed segment like the prefill's, and a
      new empty open segment follows it.

    Cluster ids: closed segments in order (the prefill's, then the closed
    appended ones), then the K open clusters.  All of a token's arithmetic
    is fp64 on the exact bf16 inputs.  Pinned by invariants (sizes sum to
    the middle count, value sums equal member sums, every open member at a
    nearest centroid with room, steady zone = first s0 and last s1 tokens),
    by equality with a one-shot build of the longer sequence when the
    segments line up, and by a hand-derived golden sequence."""

    def __init__(self, K, V, base_len: int, init_pos=None, iters: int = DEFAULT_ITERS,
                 seg_len: int = SEGMENT_TOKENS, clusters_per_seg: int = CLUSTERS_PER_SEGMENT,
                 s0: int = STEADY_INITIAL, s1: int = STEADY_RECENT, prefill: dict | None = None):
        # K, V: fp64 [N_max][d], every token the sequence will hold, by position
        self.K = np.asarray(K, dtype=np.float64)
        self.V = np.asarray(V, dtype=np.float64)
        if base_len <= s0 + s1:
            raise ValueError("the prefill must leave at least one middle token")
        self.seg_len, self.iters, self.s0, self.s1 = seg_len, iters, s0, s1
        self.Kc = min(clusters_per_seg, seg_len)
        self.N = base_len
        # the prefill's clustering: built here, or given (perm, counts,
        # offsets, centroid of another implementation's prefill index, to
        # follow its state)
        idx = prefill if prefill is not None else build_index_head(
            self.K[:base_len], self.V[:base_len], init_pos, iters, seg_len, clusters_per_seg,
            s0, s1)
        # closed clusters: members (positions, position order) and bf16 centroid
        self.members: list[list[int]] = []
        self.centroid: list[np.ndarray] = []
        self.segments: list[tuple[int, int]] = []   # (first cluster id, clusters)
        for c in range(len(idx["counts"])):
            a, n = idx["offsets"][c], idx["counts"][c]
            self.members.append([int(p) for p in idx["perm"][a:a + n]])
            self.centroid.append(idx["centroid"][c].copy())
        base = 0
        for _, _, Ks in segments(base_len - s0 - s1, seg_len, clusters_per_seg):
            self.segments.append((base, Ks))
            base += Ks
        self._open_new()

    def _open_new(self):
        first, k_last = self.segments[-1]
        self.targets = [self.centroid[first + j] for j in range(k_last)]
        self.cap = open_slots(self.seg_len, k_last)
        self.open: list[list[int]] = [[] for _ in range(self.Kc)]
        self.open_start = self._middle_end()          # first position of the open segment

    def _middle_end(self) -> int:
        return self.N - self.s1

    def open_distances(self, key: np.ndarray) -> np.ndarray:
        """||key - c_j||^2 to the last closed segment's centroids."""
        return np.array([float(((key - c) ** 2).sum()) for c in self.targets])

    def choose(self, key: np.ndarray) -> int:
        """Open cluster of a moving token: nearest target with a free slot,
        lower id on ties."""
        d = self.open_distances(key)
        room = [j for j in range(len(self.targets)) if len(self.open[j]) < self.cap]
        return min(room, key=lambda j: (d[j], j))

    def append(self, chosen: int | None = None, close_labels=None) -> dict:
        """Token N joins the sequence; token N - s1 moves into the open
        segment (to `chosen` when given: another implementation's choice,
        accepted when it has room and its distance is within 1e-5 relative of
        the nearest with room).  Closes the open segment when it is full
        (with `close_labels`, when given, as the clustering of its tokens:
        another implementation's k-means result, used to mirror its state).
        Returns {"moved": position, "cluster": open id, "closed": bool}."""
        if self.N >= self.K.shape[0]:
            raise ValueError("no more tokens to append")
        p = self.N - self.s1
        key = self.K[p]
        j = self.choose(key)
        if chosen is not None:
            d = self.open_distances(key)
            ok = (0 <= chosen < len(self.targets) and len(self.open[chosen]) < self.cap and
                  d[chosen] <= d[j] + 1e-5 * (1.0 + d[j]))
            if not ok:
                raise AssertionError(f"open cluster {chosen} is not a nearest one with room "
                                     f"(nearest {j}, distances {d[chosen]} vs {d[j]})")
            j = chosen
        self.open[j].append(p)
        self.N += 1
        closed = sum(len(m) for m in self.open) == self.seg_len
        if closed:
            self._close(close_labels)
        return dict(moved=p, cluster=j, closed=closed)

    def _close(self, labels=None):
        pos = np.arange(self.open_start, self.open_start + self.seg_len)
        X = self.K[pos]
        L, Ks = self.seg_len, self.Kc
        if labels is None:
            res = kmeans(X, strided_init(L, Ks), self.iters)
            labels, mu = res["labels"], res["mu"]
        else:
            labels = np.asarray(labels, dtype=np.int64)
            mu, _ = update(X, labels, np.zeros((Ks, X.shape[1])))
        first = len(self.members)
        for c in range(Ks):
            self.members.append([int(p) for p in pos[labels == c]])
            self.centroid.append(bf16_round(mu[c]))
        self.segments.append((first, Ks))
        self.last_labels = labels
        self._open_new()

    # ---- views
    def clusters(self) -> int:
        """Live cluster ids: the closed ones and the K open ones."""
        return len(self.members) + self.Kc

    def steady(self) -> np.ndarray:
        return steady_positions(self.N, self.s0, self.s1)

    def to_index(self) -> dict:
        """The state as an index dict for `tripartite_attention` (rows in id
        order, members in position order; open clusters beyond K_last empty
        with zero centroids)."""
        d = self.K.shape[1]
        mem = self.members + self.open
        cent = self.centroid + [self.targets[j] if j < len(self.targets) else np.zeros(d)
                                for j in range(self.Kc)]
        counts = np.array([len(m) for m in mem], dtype=np.int64)
        offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
        perm = np.array([p for m in mem for p in m], dtype=np.int64)
        vsum = np.array([self.V[m].sum(axis=0) if m else np.zeros(d) for m in mem])
        sp = self.steady()
        return dict(N=self.N, C=len(mem), perm=perm, counts=counts, offsets=offsets,
                    centroid=np.array(cent), vsum=vsum, Kp=self.K[perm], Vp=self.V[perm],
                    Ks=self.K[sp], Vs=self.V[sp])
