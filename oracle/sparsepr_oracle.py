"""Plain fp64 CPU oracle of the SparsePR sparse attention call.

TEST INFRASTRUCTURE: imported only by tests, the smoke check and the bench's
CPU-baseline leg; never by the product path.

Sources.  The method is "Partition the Support, Reconstruct the Residual:
Training-Free Sparse Attention for Video Generation and World Models"
(Taghavi, Langari, Pandey; arXiv 2608.18484), known here only through web
summaries.  Citations name the page and the paper section it summarises:

  [paperlayer §X]  paperlayer.ai section-by-section summary, section X
  [abstract]       the English abstract (paperdance.org card)
  [gist-nl §X]     gist.science Dutch technical summary, section X
                   (the Italian and Korean gist.science pages repeat it)

Numerics: every input is the bf16-rounded tensor converted to fp64; all
arithmetic is fp64.  Library primitives used as single steps: matmul,
``numpy.linalg.eigh`` (symmetric eigendecomposition), ``numpy.linalg.solve``,
``numpy.argsort`` / ``lexsort`` (stable sorts).

Readings (the pages leave these steps open; the plainest reading is taken):
  R1 sampled queries: rows floor(i*N/M_s), i < M_s.
  R2 key-response weights: top-p eigenvectors of M_K scaled by
     sqrt(lambda_i / sum_j lambda_j) (Euclidean distance in these coordinates
     is the sampled-query response-profile distance, truncated to p).
  R3 k-means init: G distinct rows from a partial Fisher-Yates shuffle driven
     by splitmix64; T Lloyd iterations, ties to the lowest index, an empty
     cluster keeps its previous centroid; labels are the T-th assignment.
  R4 query-response coordinates: u_q = s * Ctilde q over nonempty K/V groups
     (Ctilde = raw-key group means minus their unweighted mean), divided by
     sqrt(mean(u_q^2) + 1e-6).
  R5 route logit: s * qbar_i . c_j + ln|K_j| (qbar_i = mean raw query of group
     i, c_j = uncentred mean raw key of group j); cells of a query group are
     ranked by softmax mass (ties to lower j); a cell's entry mass is the
     cumulative mass ranked before it and its tail mass the mass ranked at or
     after it (1 - entry, summed from the small end so that peaked rows keep
     their tails distinct); tau mode keeps entry mass < tau; budget mode keeps
     all cells with tail mass >= the smallest value t such that the kept
     cells' true cost sum |Q_i||K_j| plus the probe pairs M*N_k fits in
     rho_target*N_q*N_k (per head); each group's top cell is always kept.
  R6 probes: one per nonempty query group, the rest apportioned by largest
     remainder on the spare capacity |Q_g|-1 (ties to lower g); if M is below
     the number of nonempty groups, the M largest groups get one each; within a
     group, members in original-index order at positions
     floor((t+1/2)|Q_g|/m_g); coverage weight (|Q_g|/m_g) normalised to sum 1.
  R7 fit: weighted (coverage weights) centring; U_r = leading eigenvectors of
     the weighted centred residual Gram (= right singular vectors), directions
     with sigma <= 1e-6 sigma_max dropped; the feature-dependent term is a
     ridge fit (absolute lambda, unpenalised intercept) of the centred
     residual's U_r coordinates on the centred sparse output, and only that
     term is restricted to U_r: the intercept keeps the full weighted mean
     residual; probe rows keep their exact dense value.
  R8 rho_exec counts routed cells and, separately, the M*N_k probe pairs.
  R11 semantic partition (the comparator of [paperlayer §2 "Token
     Partitioning"; §3.1 O3]): the R3 k-means run on the raw key rows and,
     independently, on the raw query rows, with the same initial rows,
     iteration count and tie rule; routing, hard drop, probes and the fit are
     unchanged (the pages' matched comparison).
  R12 O3 decomposition: the residual is dense minus hard-drop output over the
     rows given; its affine part is the least-squares fit of the residual on
     [sparse output, 1] (every output column jointly), the orthogonal part the
     remainder.
  R13 warm start (the pages name a warm-started GPU k-means [paperlayer App.
     C.1] and nothing more): a call's two k-means start from the previous
     call's centroids instead of seeded rows: the previous raw-key group
     means (zero for an empty group) mapped into this call's key-response
     coordinates (z = W^T k is linear, so means map by W), and the previous
     query centroids kept in head-dimension form a_g = mean of (s / rms) q,
     whose query-response coordinates are Ctilde a_g.
  R14 estimator ablation ([paperlayer §5 "Ablations", Table 4]; the pages
     do not list its rows): the unweighted estimator gives every probe the
     weight 1/M in place of the coverage weight; the estimator without the
     subspace restriction is r = d (U_r then spans the output space, so
     projecting onto it changes nothing).
  R15 O1 / O2 ([paperlayer §3.1]): a query's support at mass alpha is the
     smallest key set reaching alpha (keys ranked by probability, ties to the
     lower index); the pooled support of a set of queries is the union of
     theirs; the retained mass of a query is the attention mass on the keys
     its route keeps.
  R16 distance-ranked probes (a probe-selection variant of [paperlayer §5
     "Ablations", Table 4]): the same per-group probe counts, but each group
     takes its rows nearest its centroid in query-response coordinates
     (squared distance; ties to the lower original index).
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = [
    "Params", "attention_rows", "dense_attention", "sample_query_indices",
    "response_metric", "key_response_weights", "splitmix64_stream",
    "kmeans_init_indices", "kmeans", "kmeans_objective", "group_means",
    "kv_centroids", "query_response_coords", "group_major_permutation",
    "route_logits", "route_masses", "route_select", "route_to_csr",
    "select_probes", "hard_drop_attention", "fit_residual", "apply_correction",
    "rho_exec", "sparsepr_head", "sparsepr_call", "affine_residual_decomposition",
    "attention_probs", "minimal_support", "pooled_support", "retained_mass",
]

MASK64 = (1 << 64) - 1
RMS_EPS = 1e-6
SIGMA_DROP = 1e-6


@dataclasses.dataclass
class Params:
    """Method parameters of one call (the oracle's own copy)."""

    Ms: int
    p: int
    Gk: int
    Gq: int
    iters: int = 10
    route_mode: str = "tau"  # "tau" | "budget"
    tau: float = 0.9
    rho_target: float = 0.25
    M: int = 64
    r: int = 8
    lam: float = 1e-3
    seed: int = 0
    scale: float | None = None  # default 1/sqrt(d)
    weight_power: float = 0.5
    partition: str = "response"  # "response" | "semantic" (reading R11)
    weights: str = "coverage"  # "coverage" | "uniform" (reading R14)
    probe_select: str = "stratified"  # "stratified" | "ranked" (reading R16)


# ---------------------------------------------------------------------------
# Dense attention (the operator SparsePR approximates) [abstract]
# ---------------------------------------------------------------------------
def attention_rows(Qr, K, V, scale):
    """softmax(scale * Qr K^T) V for the given query rows, in fp64.

    Textbook softmax attention with the row maximum subtracted before exp.
    """
    S = scale * (np.asarray(Qr, np.float64) @ np.asarray(K, np.float64).T)
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=1, keepdims=True)
    return P @ np.asarray(V, np.float64)


def dense_attention(Q, K, V, scale, chunk=2048):
    """Full dense attention, row by row (rows are independent)."""
    out = np.empty((Q.shape[0], V.shape[1]), np.float64)
    for s in range(0, Q.shape[0], chunk):
        out[s:s + chunk] = attention_rows(Q[s:s + chunk], K, V, scale)
    return out


# ---------------------------------------------------------------------------
# Response-Coupled Partitioning [paperlayer §4, App. B, B.1, B.2; gist-nl §2A]
# ---------------------------------------------------------------------------
def sample_query_indices(N, Ms):
    """Deterministic sampled queries [paperlayer App. B.1]; reading R1."""
    return np.array([(i * N) // Ms for i in range(Ms)], dtype=np.int64)


def response_metric(Qs):
    """M_K = Q_s^T Q_s / M_s  [gist-nl §2A]."""
    Qs = np.asarray(Qs, np.float64)
    return Qs.T @ Qs / Qs.shape[0]


def key_response_weights(MK, p, weight_power=0.5):
    """Key-response projection W (d x p) [paperlayer App. B.1]; reading R2.

    Columns are the top-p eigenvectors of M_K (descending eigenvalue), each
    scaled by (lambda_i / sum_j lambda_j) ** weight_power.  Returns (W, lam)
    with lam the eigenvalues in descending order.
    """
    lam, U = np.linalg.eigh(np.asarray(MK, np.float64))
    order = np.argsort(-lam, kind="stable")
    lam, U = lam[order], U[:, order]
    lam = np.maximum(lam, 0.0)
    tot = lam.sum()
    wts = (lam[:p] / tot) ** weight_power if tot > 0 else np.zeros(p)
    return U[:, :p] * wts[None, :], lam


def splitmix64_stream(state):
    """splitmix64 (Steele, Lea & Flood, OOPSLA 2014): yields 64-bit outputs."""
    x = state & MASK64
    while True:
        x = (x + 0x9E3779B97F4A7C15) & MASK64
        z = x
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        yield z ^ (z >> 31)


def kmeans_init_indices(n, G, seed, bh, which):
    """G distinct row indices for k-means init (reading R3).

    Partial Fisher-Yates over 0..n-1: for i < G, j = i + (draw mod (n - i)),
    swap a[i], a[j]; the stream starts at
    seed XOR ((2*bh + which + 1) * 0xD1B54A32D192ED03) mod 2^64,
    which = 0 for keys, 1 for queries.
    """
    if G > n:
        raise ValueError("more groups than rows")
    state = (seed ^ (((2 * bh + which + 1) * 0xD1B54A32D192ED03) & MASK64)) & MASK64
    rng = splitmix64_stream(state)
    a = {}
    out = []
    for i in range(G):
        j = i + next(rng) % (n - i)
        ai, aj = a.get(i, i), a.get(j, j)
        a[i], a[j] = aj, ai
        out.append(a[i])
    return np.array(out, dtype=np.int64)


def _sqdist(X, C):
    """Squared Euclidean distances, ||x||^2 - 2 x.c + ||c||^2, fp64."""
    return (X * X).sum(1)[:, None] - 2.0 * (X @ C.T) + (C * C).sum(1)[None, :]


def kmeans(X, G, iters, init_idx=None, init_centroids=None, payload=None, payload_init=None):
    """Lloyd's k-means with a fixed iteration count (reading R3).

    Each iteration assigns every row to its nearest centroid (ties to the lower
    index; numpy's argmin returns the first minimum) and then replaces each
    centroid by the mean of its rows; an empty cluster keeps its centroid.
    The start is the rows ``init_idx`` (seeded) or ``init_centroids`` (a warm
    start, reading R13).  ``payload`` rows, if given, get the same update
    (group means under the same labels, empty groups keep theirs, starting
    from ``payload_init``): the centroids in another representation of the
    rows.  Returns (labels, centroids, objective, objective_per_iteration),
    plus the payload centroids when a payload is given.
    """
    X = np.asarray(X, np.float64)
    if init_centroids is not None:
        C = np.array(init_centroids, np.float64)
    else:
        C = X[np.asarray(init_idx)].copy()
    Pc = None
    if payload is not None:
        payload = np.asarray(payload, np.float64)
        Pc = (np.array(payload_init, np.float64) if payload_init is not None
              else payload[np.asarray(init_idx)].copy())
    lab = np.zeros(X.shape[0], np.int64)
    hist = []
    for _ in range(iters):
        lab = np.argmin(_sqdist(X, C), axis=1)
        C = group_means(X, lab, G, fallback=C)
        if payload is not None:
            Pc = group_means(payload, lab, G, fallback=Pc)
        hist.append(kmeans_objective(X, lab, C))
    res = (lab, C, (hist[-1] if hist else kmeans_objective(X, lab, C)), hist)
    return res + (Pc,) if payload is not None else res


def kmeans_objective(X, lab, C):
    """sum_n ||x_n - c_{lab_n}||^2."""
    D = np.asarray(X, np.float64) - C[lab]
    return float((D * D).sum())


def group_means(X, lab, G, fallback=None):
    """Mean row per group; groups with no rows take ``fallback`` (or NaN)."""
    X = np.asarray(X, np.float64)
    out = np.full((G, X.shape[1]), np.nan) if fallback is None else np.array(fallback, np.float64)
    for g in range(G):
        m = lab == g
        if m.any():
            out[g] = X[m].mean(axis=0)
    return out


def kv_centroids(K, lab_k, Gk):
    """Raw-key mean per K/V group and group sizes [paperlayer App. B.2]."""
    counts = np.bincount(lab_k, minlength=Gk).astype(np.int64)
    return group_means(K, lab_k, Gk), counts


def query_response_coords(Q, C, counts_k, scale, eps=RMS_EPS):
    """Query-response coordinates [paperlayer App. B.2, C.1]; reading R4.

    The logits of each query against the equally weighted, centred, nonempty
    K/V-group centroids, divided by their RMS.  Returns (U_hat, rms, Ctilde).
    """
    ne = counts_k > 0
    Cne = C[ne]
    Ct = Cne - Cne.mean(axis=0, keepdims=True)
    u = scale * (np.asarray(Q, np.float64) @ Ct.T)
    rms = np.sqrt((u * u).mean(axis=1) + eps)
    return u / rms[:, None], rms, Ct


def group_major_permutation(lab, G):
    """Stable group-major order and group offsets [paperlayer §4].

    perm[i] is the original index of the row at permuted position i; rows of
    one group keep their original relative order.
    """
    perm = np.argsort(np.asarray(lab), kind="stable")
    counts = np.bincount(lab, minlength=G)
    off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    return perm.astype(np.int64), off


# ---------------------------------------------------------------------------
# Routing [paperlayer §4 "Sparse Execution"]; reading R5
# ---------------------------------------------------------------------------
def route_logits(qbar, C, counts_k, scale):
    """Centroid logit plus log group size, over nonempty K/V groups.

    Returns an array [Gq, Gk] with -inf in columns of empty K/V groups.
    """
    Gk = C.shape[0]
    L = np.full((qbar.shape[0], Gk), -np.inf)
    ne = counts_k > 0
    L[:, ne] = scale * (qbar @ C[ne].T) + np.log(counts_k[ne].astype(np.float64))[None, :]
    return L


def route_masses(L):
    """Per query group: softmax mass of each cell, its entry and tail mass.

    Cells are ranked by mass, descending, ties to the lower K/V index.  A
    cell's entry mass e is the total mass ranked before it; its tail mass is
    the total mass ranked at or after it (1 - e in exact arithmetic), summed
    from the smallest cell upward so that tiny tails keep their relative
    precision.  Columns with -inf logits (empty K/V groups) get mass 0, entry
    mass +inf and tail 0, and are never routed.  Returns (pi, e, tail, top)
    with top marking each row's first-ranked cell.
    """
    Gq, Gk = L.shape
    pi = np.zeros((Gq, Gk))
    e = np.full((Gq, Gk), np.inf)
    tail = np.zeros((Gq, Gk))
    top = np.zeros((Gq, Gk), bool)
    for i in range(Gq):
        fin = np.isfinite(L[i])
        if not fin.any():
            continue
        row = L[i][fin] - L[i][fin].max()
        w = np.exp(row)
        w = w / w.sum()
        js = np.nonzero(fin)[0]
        order = np.lexsort((js, -w))
        ranked = w[order]
        pi[i, js] = w
        e[i, js[order]] = np.concatenate([[0.0], np.cumsum(ranked)[:-1]])
        tail[i, js[order]] = np.cumsum(ranked[::-1])[::-1]
        top[i, js[order[0]]] = True
    return pi, e, tail, top


def route_select(tail, top, counts_q, counts_k, mode, tau=0.9, rho_target=0.25, M=0):
    """Boolean cell mask [Gq, Gk]; reading R5.  Empty query groups keep none.

    Tau mode keeps cells whose entry mass is below tau, i.e. whose tail mass
    exceeds 1 - tau.  Budget mode keeps every live cell whose tail mass is at
    least t*, the smallest tail value for which the kept cells' true cost fits
    the budget rho_target*N_q*N_k - M*N_k (fp64 against integer costs).  Each
    group's top cell is always kept.
    """
    live = (counts_q > 0)[:, None] & (counts_k > 0)[None, :]
    top = top & live
    if mode == "tau":
        return (live & (tail > 1.0 - tau)) | top
    if mode != "budget":
        raise ValueError(mode)
    Nq, Nk = int(counts_q.sum()), int(counts_k.sum())
    budget = rho_target * Nq * Nk - M * Nk
    cost = counts_q[:, None].astype(np.float64) * counts_k[None, :]
    # Kept cost as a function of the threshold t is the cumulative cost of
    # live cells in descending tail order, read at the last cell with tail t;
    # it is monotone, so the feasible thresholds form a prefix.
    tv, cv = tail[live], cost[live]
    order = np.argsort(-tv, kind="stable")
    tv, cv = tv[order], cv[order]
    cum = np.cumsum(cv)
    last = np.r_[tv[1:] != tv[:-1], True] if len(tv) else np.zeros(0, bool)
    ok = np.nonzero(last & (cum <= budget))[0]
    if len(ok) == 0:
        return top
    best = tv[ok.max()]
    return (live & (tail >= best)) | top


def route_to_csr(mask):
    """CSR of selected K/V groups per query group, columns ascending."""
    row_ptr = np.concatenate([[0], np.cumsum(mask.sum(axis=1))]).astype(np.int64)
    col_idx = np.nonzero(mask)[1].astype(np.int64)  # row-major: ascending j per row
    return row_ptr, col_idx


# ---------------------------------------------------------------------------
# Probe selection [paperlayer §4, App. A.2; gist-nl §2B]; reading R6
# ---------------------------------------------------------------------------
def select_probes(counts_q, q_off, perm_q, M, dist=None):
    """Stratified probe rows and coverage weights (reading R6).

    With ``dist`` (one value per original row: its squared distance to its own
    query centroid in query-response coordinates) the m_g rows of group g are
    instead its m_g rows nearest the centroid, ties to the lower original
    index (reading R16); counts and weights are unchanged.
    Returns (probe_pos, probe_idx, weights, m_g): permuted positions, original
    row indices (both ordered by group, then position), weights summing to 1,
    and the per-group probe counts.
    """
    counts_q = np.asarray(counts_q, np.int64)
    G = counts_q.shape[0]
    N = int(counts_q.sum())
    m = np.zeros(G, np.int64)
    ne = np.nonzero(counts_q > 0)[0]
    if M > N:
        raise ValueError("more probes than rows")
    if M > 0:
        if M >= len(ne):
            m[ne] = 1
            R = M - len(ne)
            S = N - len(ne)
            if R > 0:
                num = R * (counts_q - 1)
                num[counts_q == 0] = 0
                fl = num // S
                rem = num % S
                m += fl
                left = R - int(fl.sum())
                cand = [g for g in range(G) if rem[g] > 0]
                cand.sort(key=lambda g: (-rem[g], g))
                for g in cand[:left]:
                    m[g] += 1
        else:
            order = sorted(ne.tolist(), key=lambda g: (-counts_q[g], g))
            m[order[:M]] = 1
    pos, wt = [], []
    covered = int(counts_q[m > 0].sum())
    for g in range(G):
        mg, cnt = int(m[g]), int(counts_q[g])
        if mg == 0:
            continue
        if dist is None:
            chosen = [int(q_off[g]) + ((2 * t + 1) * cnt) // (2 * mg) for t in range(mg)]
        else:
            span = np.arange(int(q_off[g]), int(q_off[g]) + cnt)
            rows = np.asarray(perm_q)[span]
            order = np.lexsort((rows, np.asarray(dist)[rows]))
            chosen = np.sort(span[order[:mg]]).tolist()
        for p_ in chosen:
            pos.append(p_)
            wt.append((counts_q[g] / m[g]) / covered)
    pos = np.array(pos, np.int64)
    return pos, np.asarray(perm_q)[pos] if len(pos) else pos, np.array(wt, np.float64), m


# ---------------------------------------------------------------------------
# Routed attention under renormalized hard drop [paperlayer §1, §4]
# ---------------------------------------------------------------------------
def hard_drop_attention(Q, K, V, lab_q, lab_k, row_ptr, col_idx, scale, rows=None):
    """Each query attends, with softmax renormalised over the retained keys,
    to the union of the K/V groups routed to its query group.

    ``rows`` restricts the output to the given original query indices (the
    result then has one row per entry of ``rows``).  Rows of a query group
    with no routed cell get zeros.
    """
    lab_q = np.asarray(lab_q)
    lab_k = np.asarray(lab_k)
    want = np.arange(Q.shape[0]) if rows is None else np.asarray(rows)
    out = np.zeros((len(want), V.shape[1]))
    gq = lab_q[want]
    for i in np.unique(gq):
        sel = np.nonzero(gq == i)[0]
        cols = col_idx[row_ptr[i]:row_ptr[i + 1]]
        if len(cols) == 0:
            continue
        keys = np.nonzero(np.isin(lab_k, cols))[0]
        out[sel] = attention_rows(Q[want[sel]], K[keys], V[keys], scale)
    return out


# ---------------------------------------------------------------------------
# Probe-Fitted Residual Reconstruction [paperlayer §4, App. A, A.3;
# gist-nl §2B]; reading R7
# ---------------------------------------------------------------------------
def fit_residual(X, D, w, r, lam, sigma_drop=SIGMA_DROP):
    """Fit the call-specific affine residual map on the probes.

    X = sparse outputs of the probes (M x d), D = their dense outputs,
    w = coverage weights (sum 1), R = D - X, Rbar = sum_t w_t R_t.
    U_r holds the leading right singular vectors of the weighted, centred
    residual W^1/2 (R - Rbar), i.e. the leading eigenvectors of its Gram
    matrix, dropping directions with sigma <= sigma_drop * sigma_max.
    The feature-dependent part is fitted inside that subspace by weighted
    ridge on centred data: B = (Xc^T W Xc + lam I)^-1 Xc^T W (Rc U_r).
    The estimator is R(x) = b + x B U_r^T with the full-width intercept
    b = Rbar - xbar B U_r^T (only the feature-dependent term is restricted).
    Returns (U, B, b, sigma): U is d x r_eff, B is d x r_eff, b has d entries,
    sigma the singular values (descending).
    """
    X = np.asarray(X, np.float64)
    R = np.asarray(D, np.float64) - X
    w = np.asarray(w, np.float64)
    d = X.shape[1]
    Rbar = w @ R
    Rc = R - Rbar
    Gram = Rc.T @ (w[:, None] * Rc)
    ev, U = np.linalg.eigh(Gram)
    order = np.argsort(-ev, kind="stable")
    ev, U = np.maximum(ev[order], 0.0), U[:, order]
    sigma = np.sqrt(ev)
    keep = 0
    if sigma[0] > 0:
        keep = int(min(r, np.count_nonzero(sigma > sigma_drop * sigma[0])))
    U = U[:, :keep]
    xbar = w @ X
    Xc = X - xbar
    Yc = Rc @ U
    A = Xc.T @ (w[:, None] * Xc) + lam * np.eye(d)
    B = np.linalg.solve(A, Xc.T @ (w[:, None] * Yc))
    b = Rbar - (xbar @ B) @ U.T
    return U, B, b, sigma


def apply_correction(X, U, B, b):
    """Estimated dense rows: x + b + x B U^T  [gist-nl §2B "Correctie"]."""
    X = np.asarray(X, np.float64)
    return X + b[None, :] + (X @ B) @ U.T


def rho_exec(counts_q, counts_k, row_ptr, col_idx, M):
    """Executed-pair density including probe rows [paperlayer §4, App. C.3].

    Returns (routed_pairs, probe_pairs, rho).
    """
    routed = 0
    for i in range(len(counts_q)):
        for j in col_idx[row_ptr[i]:row_ptr[i + 1]]:
            routed += int(counts_q[i]) * int(counts_k[j])
    Nq, Nk = int(np.sum(counts_q)), int(np.sum(counts_k))
    probe = int(M) * Nk
    return routed, probe, (routed + probe) / (Nq * Nk)


# ---------------------------------------------------------------------------
# Whole call
# ---------------------------------------------------------------------------
def sparsepr_head(Q, K, V, prm: Params, bh=0, lab_k=None, lab_q=None, csr=None,
                  rows=None, want_dense=False, warm=None, probe_pos=None):
    """One (batch, head) SparsePR call, fp64, following the pages' order.

    Driven mode: ``lab_k`` / ``lab_q`` (and optionally ``csr``) replace the
    oracle's own clustering (routing) so that everything downstream is
    recomputed from given assignments; ``probe_pos`` likewise replaces the
    selected probe positions (ascending, with the selection's own per-group
    counts; for ranked selection, where rows whose distances tie at the cut
    may be taken either way).  ``rows`` limits the routed attention
    and the output to those original rows (probe rows are always computed).
    ``warm`` (reading R13) is the ``warm_state`` a previous call returned:
    both k-means then start from its centroids instead of seeded rows.
    Returns a dict of every intermediate.
    """
    Q = np.asarray(Q, np.float64)
    K = np.asarray(K, np.float64)
    V = np.asarray(V, np.float64)
    N, d = Q.shape
    s = prm.scale if prm.scale is not None else 1.0 / np.sqrt(d)
    out = {"scale": s}
    if prm.partition == "semantic":
        # Semantic comparator (reading R11): k-means on the raw rows
        a_q = None
        if lab_k is None:
            init_k = kmeans_init_indices(K.shape[0], prm.Gk, prm.seed, bh, 0)
            lab_k, _, _, hist_k = kmeans(K, prm.Gk, prm.iters, init_k,
                                         init_centroids=None if warm is None else warm["C_raw"])
            out["kmeans_k_hist"] = hist_k
        lab_k = np.asarray(lab_k, np.int64)
        C, counts_k = kv_centroids(K, lab_k, prm.Gk)
        out["obj_k"] = kmeans_objective(K, lab_k, np.where((counts_k > 0)[:, None], C, 0.0))
        if lab_q is None:
            init_q = kmeans_init_indices(N, prm.Gq, prm.seed, bh, 1)
            lab_q, a_q, _, hist_q = kmeans(Q, prm.Gq, prm.iters, init_q,
                                           init_centroids=None if warm is None else warm["a_q"])
            out["kmeans_q_hist"] = hist_q
        lab_q = np.asarray(lab_q, np.int64)
        Cu = group_means(Q, lab_q, prm.Gq)
        ne_q = np.bincount(lab_q, minlength=prm.Gq) > 0
        out["obj_q"] = kmeans_objective(Q, lab_q, np.where(ne_q[:, None], Cu, 0.0))
        rms, Ct = None, None
        Xq = Q
    else:
        # Key-response coordinates and paired K/V groups
        qs_idx = sample_query_indices(N, prm.Ms)
        MK = response_metric(Q[qs_idx])
        W, lamk = key_response_weights(MK, prm.p, prm.weight_power)
        Z = K @ W
        out.update(MK=MK, W=W, eig_MK=lamk, Z=Z)
        a_q = None
        if lab_k is None:
            init_k = kmeans_init_indices(K.shape[0], prm.Gk, prm.seed, bh, 0)
            # warm start: the previous raw-key means in today's coordinates
            # (z = W^T k is linear, so a group mean maps by W as well)
            lab_k, _, _, hist_k = kmeans(
                Z, prm.Gk, prm.iters, init_k,
                init_centroids=None if warm is None else np.asarray(warm["C_raw"]) @ W)
            out["kmeans_k_hist"] = hist_k
        lab_k = np.asarray(lab_k, np.int64)
        Cz = group_means(Z, lab_k, prm.Gk)
        ne_k = np.bincount(lab_k, minlength=prm.Gk) > 0
        out["obj_k"] = kmeans_objective(Z, lab_k, np.where(ne_k[:, None], Cz, 0.0))
        C, counts_k = kv_centroids(K, lab_k, prm.Gk)
        # Query-response coordinates and query groups
        Uq, rms, Ct = query_response_coords(Q, C, counts_k, s)
        if lab_q is None:
            init_q = kmeans_init_indices(N, prm.Gq, prm.seed, bh, 1)
            # the centroids are carried along in head-dimension form as the
            # means of (s / rms) q (u = s Ctilde q / rms, so m = Ctilde a):
            # that form is what survives to the next call's coordinates
            Qf = (s / rms)[:, None] * Q
            a0 = None if warm is None else np.asarray(warm["a_q"])
            lab_q, _, _, hist_q, a_q = kmeans(
                Uq, prm.Gq, prm.iters, init_q,
                init_centroids=None if a0 is None else a0 @ Ct.T, payload=Qf, payload_init=a0)
            out["kmeans_q_hist"] = hist_q
        lab_q = np.asarray(lab_q, np.int64)
        Cu = group_means(Uq, lab_q, prm.Gq)
        ne_q = np.bincount(lab_q, minlength=prm.Gq) > 0
        out["obj_q"] = kmeans_objective(Uq, lab_q, np.where(ne_q[:, None], Cu, 0.0))
        Xq = Uq
    out.update(lab_k=lab_k, lab_q=lab_q, C=C, counts_k=counts_k, rms=rms, Ctilde=Ct,
               Cu=Cu)
    # what a warm-started next call starts from (reading R13): raw-key group
    # means (zero for an empty group) and the query centroids in head-dim form
    out["warm_state"] = {"C_raw": np.where((counts_k > 0)[:, None], np.nan_to_num(C), 0.0),
                         "a_q": a_q}
    # Group-major layouts
    perm_k, kv_off = group_major_permutation(lab_k, prm.Gk)
    perm_q, q_off = group_major_permutation(lab_q, prm.Gq)
    counts_q = np.bincount(lab_q, minlength=prm.Gq).astype(np.int64)
    qbar = group_means(Q, lab_q, prm.Gq)
    out.update(perm_k=perm_k, kv_off=kv_off, perm_q=perm_q, q_off=q_off,
               counts_q=counts_q, qbar=qbar)
    # Routing
    L = route_logits(np.nan_to_num(qbar), C, counts_k, s)
    pi, e, tail, top = route_masses(L)
    if csr is None:
        mask = route_select(tail, top, counts_q, counts_k, prm.route_mode, prm.tau,
                            prm.rho_target, prm.M)
        row_ptr, col_idx = route_to_csr(mask)
    else:
        row_ptr, col_idx = (np.asarray(a, np.int64) for a in csr)
    out.update(route_logits=L, route_pi=pi, route_entry=e, route_tail=tail, row_ptr=row_ptr,
               col_idx=col_idx)
    # Probes
    dist = None
    if prm.probe_select == "ranked":  # reading R16: nearest to the own query centroid
        dist = ((Xq - Cu[lab_q]) ** 2).sum(axis=1)
        out["probe_dist"] = dist
        out["probe_u2"] = (Xq * Xq).sum(axis=1)  # ||u||^2, the scale of a fp32 evaluation
    probe_pos, probe_idx, wts, m_g = select_probes(counts_q, q_off, perm_q, prm.M, dist)
    if probe_pos is not None:  # driven: another valid choice of the same per-group counts
        given = np.asarray(probe_pos, np.int64)
        grp = np.searchsorted(np.asarray(q_off, np.int64), given, side="right") - 1
        if (len(given) != len(probe_pos) or (np.diff(given) <= 0).any()
                or not (np.bincount(grp, minlength=prm.Gq) == m_g).all()):
            raise ValueError("driven probe positions do not match the per-group counts")
        probe_pos, probe_idx = given, np.asarray(perm_q)[given]
    if prm.weights == "uniform" and len(wts):  # the unweighted estimator (reading R14)
        wts = np.full(len(wts), 1.0 / len(wts))
    routed, probe_pairs, rho = rho_exec(counts_q, counts_k, row_ptr, col_idx, prm.M)
    out.update(probe_pos=probe_pos, probe_idx=probe_idx, probe_w=wts, probe_m=m_g,
               routed_pairs=routed, probe_pairs=probe_pairs, rho_exec=rho)
    # Sparse execution and exact probe rows
    want = np.arange(N) if rows is None else np.asarray(rows, np.int64)
    O_sp = hard_drop_attention(Q, K, V, lab_q, lab_k, row_ptr, col_idx, s, rows=want)
    out["rows"] = want
    out["O_sp"] = O_sp
    if prm.M > 0:
        X = hard_drop_attention(Q, K, V, lab_q, lab_k, row_ptr, col_idx, s, rows=probe_idx)
        Dn = attention_rows(Q[probe_idx], K, V, s)
        U, B, b, sig = fit_residual(X, Dn, wts, prm.r, prm.lam)
        O = apply_correction(O_sp, U, B, b)
        is_probe = np.isin(want, probe_idx)
        where = {int(t): k for k, t in enumerate(probe_idx)}
        for k in np.nonzero(is_probe)[0]:
            O[k] = Dn[where[int(want[k])]]
        out.update(probe_sparse=X, probe_dense=Dn, U=U, B=B, b=b, sigma=sig)
    else:
        O = O_sp.copy()
    out["O"] = O
    if want_dense:
        out["O_dense"] = dense_attention(Q[want], K, V, s)
    return out


def affine_residual_decomposition(O_sparse, O_dense):
    """O3 diagnostic [paperlayer §3.1 O3]; reading R12.

    R = O_dense - O_sparse.  Its affine part P is the least-squares fit of R
    on the features [O_sparse, 1] (one coefficient matrix for all output
    columns), the orthogonal part E = R - P.  Returns a dict with the
    residual, affine and orthogonal energies (squared Frobenius norms) and the
    affine-explainable fraction ||P||^2 / ||R||^2.  It needs the full dense
    residual, so it is a diagnostic of a partition, not part of execution.
    """
    X = np.asarray(O_sparse, np.float64)
    R = np.asarray(O_dense, np.float64) - X
    F = np.concatenate([X, np.ones((X.shape[0], 1))], axis=1)
    beta, *_ = np.linalg.lstsq(F, R, rcond=None)
    P = F @ beta
    E = R - P
    er, ep, eo = float((R * R).sum()), float((P * P).sum()), float((E * E).sum())
    return {"residual_energy": er, "affine_energy": ep, "orthogonal_energy": eo,
            "affine_fraction": ep / er if er > 0 else 0.0}


def attention_probs(Qr, K, scale):
    """Softmax attention probabilities of query rows Qr over all keys, fp64."""
    S = scale * (np.asarray(Qr, np.float64) @ np.asarray(K, np.float64).T)
    S -= S.max(axis=1, keepdims=True)
    P = np.exp(S)
    return P / P.sum(axis=1, keepdims=True)


def minimal_support(p, alpha):
    """O1 [paperlayer §3.1 O1]; reading R15.  The smallest key set of one
    query reaching attention mass alpha: keys ranked by probability (ties to
    the lower index), taken until the running mass reaches alpha."""
    p = np.asarray(p, np.float64)
    order = np.lexsort((np.arange(len(p)), -p))
    k = int(np.searchsorted(np.cumsum(p[order]), alpha * p.sum(), side="left")) + 1
    return np.sort(order[:min(k, len(p))])


def pooled_support(P, alpha):
    """O1: per-query minimal supports of the rows of P and their union (the
    support a shared route must cover for these queries), as fractions of the
    keys.  Returns (per_query_fractions, pooled_fraction)."""
    P = np.asarray(P, np.float64)
    sets = [minimal_support(row, alpha) for row in P]
    per = np.array([len(s_) for s_ in sets], np.float64) / P.shape[1]
    pooled = len(np.unique(np.concatenate(sets))) / P.shape[1]
    return per, pooled


def retained_mass(P, keep):
    """O2 [paperlayer §3.1 O2]: attention mass each query keeps under a key
    mask (rows of ``keep`` are the kept keys of each query)."""
    return (np.asarray(P, np.float64) * np.asarray(keep, bool)).sum(axis=1)


def sparsepr_call(Q, K, V, prm: Params, **kw):
    """All heads of a [B, H, N, d] call; returns a list of per-head dicts.

    Keyword arrays given per head (lab_k, lab_q, csr, rows) are lists indexed
    by flat head index b*H + h.
    """
    Bn, Hn = Q.shape[:2]
    res = []
    for b in range(Bn):
        for h in range(Hn):
            bh = b * Hn + h
            per = {k: (v[bh] if v is not None else None) for k, v in kw.items()
                   if k in ("lab_k", "lab_q", "csr", "rows")}
            other = {k: v for k, v in kw.items() if k not in per}
            res.append(sparsepr_head(Q[b, h], K[b, h], V[b, h], prm, bh=bh, **per, **other))
    return res
