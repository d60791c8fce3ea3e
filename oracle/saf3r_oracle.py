"""CPU oracle for head-wise dynamic sparse global attention (test infrastructure).

This is the plain, slow, fp64 statement of what the SAF3R method computes
("SAF3R: Dynamic Sparse Attention for Feed-Forward 3D Reconstruction
Transformers", arXiv 2607.03612).  Only the test suite, the smoke check and the
CPU-baseline leg of the benchmark may import it; the library never does, and it
shares no code with the CUDA path.  Inputs are the exact values of the bf16
tensors (as fp32 or fp64 numpy arrays); every reduction runs in fp64.  Where the
method turns a floating-point score into a selection (probe Top-K, tile
Top-K), the score is rounded once to fp32 and ranked in fp32, the precision the
CUDA kernels rank in, with ties going to the lower index.

Section references below are to that paper unless another page is named:
  * section 4.1 "Tailored Sparse Attention Kernels" (static, query-probe Top-K,
    DINO Top-K and uniform-sampling kernels; each keeps every query and restricts
    the keys),
  * section 4.2 "Offline Head Profiling" (eq. 1, the output NMSE, and eq. 2, the
    cost-constrained choice),
  * section 4.3 "Online Pattern Adaptation" (mean-query probe; block-wise DINO
    similarity cached per input).

Readings where the pages leave a step open (each also listed in the design
notes): token layout = per view 5 special tokens then raster patches; the
static "same cell +/-1" pattern = 3x3 Chebyshev neighbourhood clipped at the
grid edge, plus every special token and every token of anchor view 0; the
stride lattice runs over the flat token index with phase = head mod stride;
the probe ranks patch keys only and the special tokens are always kept; the
block-wise DINO similarity is the cosine of per-tile means of L2-normalised
patch features over flat 64-token tiles, own tile included; excluded keys get
logit -inf (exact renormalised softmax over the kept set).

Parity status: every function here is pinned by tests in
tests/test_oracle_pins.py.  `nmse_table_sampled` is pinned on all rows against
per-row terms built from torch's fp64 SDPA, and its row-sample estimate by its
sampling distribution (within 6 standard errors of the all-row value); at the
full sizes the GPU tests use, only the sample estimate is computed.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence

import numpy as np

POSITION, PROBE, CORR, SCAN, DENSE, HYBRID, TOKEN = 0, 1, 2, 3, 4, 5, 6


# ----------------------------------------------------------------------------
# token layout
# ----------------------------------------------------------------------------

def token_parts(L, t):
    """(view, local index) of token t; local < n_special is a special token."""
    return t // L.V, t % L.V


def is_special(L, t) -> np.ndarray:
    return (np.asarray(t) % L.V) < L.n_special


def special_tokens(L) -> np.ndarray:
    """All special tokens of all views, ascending."""
    return np.array([s * L.V + i for s in range(L.S) for i in range(L.n_special)], dtype=np.int64)


def patch_tokens(L) -> np.ndarray:
    t = np.arange(L.N, dtype=np.int64)
    return t[~is_special(L, t)]


# ----------------------------------------------------------------------------
# key sets of the four kernels (section 4.1)
# ----------------------------------------------------------------------------

def position_set(L, i: int, radius: int = 1) -> np.ndarray:
    """Static kernel (section 4.1, "Static Kernel"): a fixed, content-free set.

    Query i keeps every special token, every token of the anchor view 0, and,
    when i is a patch token at grid cell (r, c), the cells (r+dr, c+dc) with
    |dr|, |dc| <= radius of every view (clipped at the grid border, no wrap).
    radius = -1 keeps the anchor frame (and the specials) only.
    """
    keys = set(special_tokens(L).tolist())
    keys.update(range(0, L.V))
    s, loc = token_parts(L, int(i))
    if loc >= L.n_special:
        r, c = divmod(loc - L.n_special, L.g)
        for sv in range(L.S):
            for rr in range(r - radius, r + radius + 1):
                if rr < 0 or rr >= L.g:
                    continue
                for cc in range(c - radius, c + radius + 1):
                    if 0 <= cc < L.g:
                        keys.add(sv * L.V + L.n_special + rr * L.g + cc)
    return np.array(sorted(keys), dtype=np.int64)


def stride_set(L, stride: int, phase: int) -> np.ndarray:
    """Uniform sampling kernel (section 4.1): keys at a fixed stride over the
    flat token index, {j : j mod stride == phase}, plus every special token."""
    j = np.arange(L.N, dtype=np.int64)
    keep = (j % stride == phase) | is_special(L, j)
    return j[keep]


def probe_mean(Qh: np.ndarray, accum=np.float64) -> np.ndarray:
    """Mean query over all N queries (section 4.3, "Query-Probe Top-K Kernel"):
    qbar = (1/N) sum_i q_i, summed in fp64 (or `accum`) and rounded once to fp32."""
    q = np.asarray(Qh, dtype=accum)
    return (q.sum(axis=0) / accum(q.shape[0])).astype(np.float32)


def probe_scores(qbar32: np.ndarray, Kh: np.ndarray, accum=np.float64) -> np.ndarray:
    """Probe score of every key, qbar K^T / sqrt(D) (section 4.3), in fp64 (or
    `accum`) and rounded to fp32 (the precision the selection is taken in)."""
    k = np.asarray(Kh, dtype=accum)
    d = k.shape[1]
    return ((k @ qbar32.astype(accum)) / accum(math.sqrt(d))).astype(np.float32)


def topk_desc(scores: np.ndarray, k: int, candidates: np.ndarray | None = None) -> np.ndarray:
    """The k best candidates by (score descending, index ascending), in rank order."""
    if candidates is None:
        candidates = np.arange(len(scores), dtype=np.int64)
    cand = np.asarray(candidates, dtype=np.int64)
    sc = np.asarray(scores)[cand]
    order = np.lexsort((cand, -sc.astype(np.float64)))
    return cand[order[:k]]


def probe_topk(L, scores32: np.ndarray, k: int) -> np.ndarray:
    """Top-K patch keys by probe score (ties to the lower index), ascending."""
    return np.sort(topk_desc(scores32, k, patch_tokens(L)))


def probe_set(L, probe_keys: np.ndarray) -> np.ndarray:
    """Key set of a vertical-line head: the probe's keys plus every special token."""
    return np.union1d(probe_keys, special_tokens(L)).astype(np.int64)


def dino_tile_means(L, dino: np.ndarray, accum=np.float64) -> np.ndarray:
    """Block-wise DINO descriptors (section 4.3, "DINO Top-K Kernel", block-wise
    variant): for each flat 64-token tile t = [64t, 64t+64) of the token
    sequence, the mean over its patch tokens of the L2-normalised DINO features
    (special tokens carry no DINO feature).  fp64 (or `accum`) [T][dino_dim]."""
    f = np.asarray(dino, dtype=accum)
    f = f / np.linalg.norm(f, axis=1, keepdims=True)
    out = np.zeros((L.T, f.shape[1]), dtype=accum)
    for t in range(L.T):
        toks = np.arange(t * L.tile, min((t + 1) * L.tile, L.N), dtype=np.int64)
        toks = toks[~is_special(L, toks)]
        if len(toks) == 0:
            continue
        s, loc = token_parts(L, toks)
        rows = s * L.P + (loc - L.n_special)
        out[t] = f[rows].mean(axis=0)
    return out


def tile_cosines(means: np.ndarray) -> np.ndarray:
    """Cosine similarity between every pair of tile descriptors, in the descriptors'
    precision (fp64 unless the selection runs with fp32 accumulation) -> fp32."""
    nrm = np.linalg.norm(means, axis=1)
    cos = (means @ means.T) / np.outer(nrm, nrm)
    return cos.astype(np.float32)


def tile_topk(cos32: np.ndarray, kt: int) -> np.ndarray:
    """For each query tile u, the kt key tiles of highest cosine (own tile
    included; ties to the lower tile index), in rank order.  int64 [T][kt]."""
    T = cos32.shape[0]
    out = np.empty((T, kt), dtype=np.int64)
    for u in range(T):
        out[u] = topk_desc(cos32[u], kt)
    return out


def tile_tokens(L, v: int) -> np.ndarray:
    return np.arange(v * L.tile, min((v + 1) * L.tile, L.N), dtype=np.int64)


def corr_set(L, tiles: Sequence[int]) -> np.ndarray:
    """Key set of a correspondence head for the queries of one tile: the tokens
    of its selected key tiles plus every special token, each key once."""
    parts = [tile_tokens(L, int(v)) for v in tiles] + [special_tokens(L)]
    return np.unique(np.concatenate(parts))


def unit_features(dino: np.ndarray, accum=np.float64) -> np.ndarray:
    """L2-normalised DINO features of the patch tokens, fp64 (or `accum`) [S*P][dim]."""
    f = np.asarray(dino, dtype=accum)
    return f / np.linalg.norm(f, axis=1, keepdims=True)


def token_topk_row(L, unit: np.ndarray, i: int, k: int) -> np.ndarray:
    """Token-wise DINO Top-K (section 4.1, "DINO Top-K Kernel"; section 5.1: K per frame): for the
    patch query token i, in every frame s the k patch tokens of highest cosine (fp64 dot of unit
    features, rounded to fp32; its own token included; ties to the lower patch index), in rank
    order, as patch indices.  int64 [S][k]."""
    s_i, loc = token_parts(L, int(i))
    a = s_i * L.P + (loc - L.n_special)
    cos32 = (unit @ unit[a]).astype(np.float32)
    out = np.empty((L.S, k), dtype=np.int64)
    for sv in range(L.S):
        out[sv] = topk_desc(cos32[sv * L.P:(sv + 1) * L.P], k)
    return out


def token_set(L, unit: np.ndarray, i: int, k: int, lists: np.ndarray | None = None) -> np.ndarray:
    """Key set of a token-wise correspondence head for query i: the per-frame Top-K patch tokens
    plus every special token; a special-token query (no DINO feature) keeps every key.
    `lists` ([S*P][S][>=k] patch indices per query and frame) replaces the ranking when given:
    a set that another ranking produced and that was found valid (equal to this one's up to keys
    tied within the boundary band), whose attention is then evaluated exactly."""
    s_i, loc = token_parts(L, int(i))
    if loc < L.n_special:
        return np.arange(L.N, dtype=np.int64)
    if lists is None:
        p = token_topk_row(L, unit, i, k)
    else:
        p = np.asarray(lists[s_i * L.P + (loc - L.n_special)], dtype=np.int64)[:, :k]
    toks = (np.arange(L.S, dtype=np.int64)[:, None] * L.V + L.n_special + p).ravel()
    return np.union1d(toks, special_tokens(L)).astype(np.int64)


# ----------------------------------------------------------------------------
# attention (section 4.1: exact softmax over the kept keys)
# ----------------------------------------------------------------------------

def attention_weights(q: np.ndarray, K: np.ndarray) -> np.ndarray:
    """softmax_j(q . k_j / sqrt(d)) over the given keys, fp64.  Keys not passed
    in are excluded, which equals giving them logit -inf."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    logits = (K @ q.T).T / math.sqrt(K.shape[1])
    logits = np.atleast_2d(logits)
    m = logits.max(axis=1, keepdims=True)
    w = np.exp(logits - m)
    return w / w.sum(axis=1, keepdims=True)


def attention_rows(q: np.ndarray, K: np.ndarray, V: np.ndarray) -> np.ndarray:
    """O = softmax(q K^T / sqrt(d)) V for a batch of query rows sharing one key set."""
    w = attention_weights(np.atleast_2d(q), K)
    return w @ np.asarray(V, dtype=np.float64)


def dense_rows(Qh, Kh, Vh, rows) -> np.ndarray:
    """Full attention O_full (section 4.2) for the given query rows."""
    return attention_rows(np.asarray(Qh)[rows], Kh, Vh)


# ----------------------------------------------------------------------------
# whole-layer selection and evaluation
# ----------------------------------------------------------------------------

class Selection:
    """The per-input index state of one layer: probe keys per probe head and the
    ranked tile list of the correspondence heads (section 4.3, index caching)."""

    def __init__(self):
        self.probe_keys: Dict[int, np.ndarray] = {}
        self.probe_scores: Dict[int, np.ndarray] = {}
        self.tile_rank: np.ndarray | None = None
        self.unit: np.ndarray | None = None  # unit DINO features (token-wise heads; their sets are computed per row)
        self.tile_cos: np.ndarray | None = None
        # per token-wise head, given per-frame lists [S*P][S][k] that replace the ranking (see token_set)
        self.token_lists: Dict[int, np.ndarray] = {}


def select(L, heads, Q, K, dino, accum=np.float64) -> Selection:
    """Build the dynamic index sets of one input (section 4.3).  `accum` = np.float32
    runs every reduction in fp32 instead of fp64, to show that the index sets do not
    hinge on the accumulation precision (they may differ only at near-ties of the
    k-th score)."""
    sel = Selection()
    kt_max = 0
    for h, hc in enumerate(heads):
        if hc.kind == PROBE:
            qbar = probe_mean(Q[h], accum)
            sc = probe_scores(qbar, K[h], accum)
            sel.probe_scores[h] = sc
            sel.probe_keys[h] = probe_topk(L, sc, hc.k)
        elif hc.kind in (CORR, HYBRID):
            kt_max = max(kt_max, hc.k)
        elif hc.kind == TOKEN and sel.unit is None:
            sel.unit = unit_features(dino, accum)
    if kt_max > 0:
        cos = tile_cosines(dino_tile_means(L, dino, accum))
        sel.tile_cos = cos
        sel.tile_rank = tile_topk(cos, kt_max)
    return sel


def key_set(L, hc, sel: Selection, h: int, i: int) -> np.ndarray:
    """Kept keys of query i under head configuration hc."""
    if hc.kind == POSITION:
        return position_set(L, i, hc.radius)
    if hc.kind == PROBE:
        return probe_set(L, sel.probe_keys[h])
    if hc.kind == SCAN:
        return stride_set(L, hc.stride, hc.phase)
    if hc.kind == CORR:
        return corr_set(L, sel.tile_rank[i // L.tile, :hc.k])
    if hc.kind == HYBRID:
        # section 5.3 ("Further Analysis of the DINO Top-K kernel"): the DINO tiles combined
        # with uniform striding, i.e. the union of the two kept sets
        return np.union1d(corr_set(L, sel.tile_rank[i // L.tile, :hc.k]), stride_set(L, hc.stride, hc.phase))
    if hc.kind == TOKEN:
        return token_set(L, sel.unit, i, hc.k, sel.token_lists.get(h))
    if hc.kind == DENSE:
        return np.arange(L.N, dtype=np.int64)
    raise ValueError(hc.kind)


def _group_key(L, hc, i: int):
    """Rows with equal group keys have equal key sets (used only to batch rows)."""
    if hc.kind in (PROBE, SCAN, DENSE):
        return 0
    if hc.kind in (CORR, HYBRID):
        return i // L.tile
    if hc.kind == TOKEN:  # every patch query has its own set; special queries keep every key
        s, loc = token_parts(L, i)
        return -1 if loc < L.n_special else i
    s, loc = token_parts(L, i)
    return -1 if loc < L.n_special else loc


def sparse_rows(L, hc, sel: Selection, h: int, Qh, Kh, Vh, rows) -> np.ndarray:
    """Sparse attention output (fp64) of the given query rows of head h."""
    rows = np.asarray(rows, dtype=np.int64)
    out = np.empty((len(rows), Qh.shape[1]), dtype=np.float64)
    groups: Dict[object, List[int]] = {}
    for n, i in enumerate(rows):
        groups.setdefault(_group_key(L, hc, int(i)), []).append(n)
    for _, idx in groups.items():
        keys = key_set(L, hc, sel, h, int(rows[idx[0]]))
        out[idx] = attention_rows(np.asarray(Qh)[rows[idx]], np.asarray(Kh)[keys], np.asarray(Vh)[keys])
    return out


def kept_count(L, hc, sel: Selection, h: int, i: int) -> int:
    return len(key_set(L, hc, sel, h, i))


def kept_pairs(L, hc, sel: Selection, h: int) -> int:
    """Exact number of (query, kept key) pairs of a head over all N queries."""
    if hc.kind == TOKEN:
        # per patch query S*k patch keys (distinct frames are disjoint) + the specials; special
        # queries every key (the per-row sets agree with this count: tests/test_oracle_pins.py)
        nsp = L.S * L.n_special
        return L.S * L.P * (L.S * hc.k + nsp) + nsp * L.N
    total = 0
    seen: Dict[object, int] = {}
    for i in range(L.N):
        g = _group_key(L, hc, i)
        if g not in seen:
            seen[g] = kept_count(L, hc, sel, h, i)
        total += seen[g]
    return total


def omega(L, pairs: int) -> int:
    """Computational cost of a configuration in FLOPs (section 4.2, Omega(c)):
    attention FLOPs only, 2d for q.k and 2d for p.v per kept pair."""
    return 4 * L.d * int(pairs)


# ----------------------------------------------------------------------------
# profiling (section 4.2)
# ----------------------------------------------------------------------------

def nmse(O_full: np.ndarray, O_sparse: np.ndarray) -> float:
    """Eq. 1 for one input: ||O_full - O_sparse||^2 / ||O_full||^2 (fp64)."""
    a = np.asarray(O_full, dtype=np.float64)
    b = np.asarray(O_sparse, dtype=np.float64)
    return float(((a - b) ** 2).sum() / (a ** 2).sum())


def choose_config(nmse_row: Sequence[float], omega_row: Sequence[int], nmse_max: float) -> int:
    """Per-head choice of the profiled stack: the cheapest candidate (minimum
    Omega, ties to the lower candidate index) whose NMSE is at most nmse_max;
    if no candidate qualifies, the one of least NMSE (the eq. 2 argmin; ties to
    the lower index)."""
    ok = [c for c in range(len(nmse_row)) if nmse_row[c] <= nmse_max]
    if ok:
        return min(ok, key=lambda c: (omega_row[c], c))
    return min(range(len(nmse_row)), key=lambda c: (nmse_row[c], c))


def baseline_stride(sigma: float) -> int:
    """Stride of the uniform-sampling baseline with sparsity at least sigma (section 4.2 starts
    the search from uniform sampling at sparsity ratio sigma; section 5.1 uses sigma = 0.85):
    keeping one key in s gives sparsity 1 - 1/s >= sigma for s = ceil(1 / (1 - sigma))."""
    s = 1
    while 1.0 - 1.0 / s < sigma - 1e-12:
        s += 1
    return s


def choose_eq2(nmse_tables, pairs_tables, base: int) -> List[int]:
    """Section 4.2, eq. 2 by progressive substitution: eq. 1 averaged over the calibration
    inputs, cost Omega = 4*d*mean(kept pairs).  Per head, start from the baseline candidate;
    walk the candidates in order and substitute c whenever it costs no more than the
    baseline and its averaged NMSE is lower than the current choice's."""
    E = np.mean(np.asarray(nmse_tables, dtype=np.float64), axis=0)
    W = np.mean(np.asarray(pairs_tables, dtype=np.float64), axis=0)
    H, C = E.shape
    out = []
    for h in range(H):
        cur = base
        for c in range(C):
            if c != base and W[h, c] <= W[h, base] and E[h, c] < E[h, cur]:
                cur = c
        out.append(cur)
    return out


def apply_candidate(hc, h: int):
    """A candidate applied to head h: scan and hybrid candidates take phase = h mod stride."""
    if hc.kind in (SCAN, HYBRID):
        return type(hc)(hc.kind, k=hc.k, stride=hc.stride, phase=h % hc.stride, radius=hc.radius)
    return hc


def nmse_table_sampled(L, candidates, Q, K, V, dino, rows_per_head) -> np.ndarray:
    """NMSE of every (head, candidate) estimated on sampled query rows.

    With all rows this is exactly eq. 1 for one calibration input; with a row
    sample it is the ratio estimate of it over those rows."""
    H = Q.shape[0]
    table = np.zeros((H, len(candidates)), dtype=np.float64)
    full = [dense_rows(Q[h], K[h], V[h], rows_per_head[h]) for h in range(H)]  # O_full, once per head
    for c, cand in enumerate(candidates):
        heads = [apply_candidate(cand, h) for h in range(H)]
        sel = select(L, heads, Q, K, dino)
        for h in range(H):
            os_ = sparse_rows(L, heads[h], sel, h, Q[h], K[h], V[h], rows_per_head[h])
            table[h, c] = nmse(full[h], os_)
    return table
