"""Comparison helpers of the GPU parity tests (test code only)."""
import copy

import numpy as np

import oracle as O

# tolerances of the GPU path against the oracle (bf16 inputs, fp32 accumulation)
MAX_ABS = 1e-2
REL_L2 = 5e-3
BOUNDARY_REL = 1e-5


def compare_outputs(gpu: np.ndarray, ref: np.ndarray, what: str):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    err = np.abs(gpu - ref)
    rel = np.linalg.norm(gpu - ref) / max(np.linalg.norm(ref), 1e-300)
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e} > {MAX_ABS}"
    assert rel <= REL_L2, f"{what}: rel-L2 {rel:.3e} > {REL_L2}"
    return float(err.max()), float(rel)


def check_topk_set(gpu_keys, ref_ranked, scores, k, what):
    """gpu_keys: the GPU's kept set; ref_ranked: the oracle's candidates in rank order
    (at least k); scores: oracle fp32 score per candidate id.  The sets must agree
    except for keys whose score is within BOUNDARY_REL of the k-th score.
    Returns True when the sets are identical."""
    g = set(int(x) for x in np.asarray(gpu_keys).tolist())
    r = set(int(x) for x in np.asarray(ref_ranked[:k]).tolist())
    assert len(g) == k, f"{what}: {len(g)} distinct keys, expected {k}"
    if g == r:
        return True
    kth = float(scores[int(ref_ranked[k - 1])])
    tol = BOUNDARY_REL * max(abs(kth), 1e-30)
    for x in g ^ r:
        assert abs(float(scores[x]) - kth) <= tol, \
            f"{what}: key {x} score {float(scores[x])!r} vs k-th {kth!r} outside the boundary band"
    return False


def check_probe(gpu_keys, L, sel, h, k, what):
    ranked = O.topk_desc(sel.probe_scores[h], k + 8, O.patch_tokens(L))
    return check_topk_set(gpu_keys, ranked, sel.probe_scores[h], k, what)


def check_tiles(gpu_ranked, sel, k, what):
    """gpu_ranked: int [T][k] from the cache export."""
    T = sel.tile_cos.shape[0]
    exact = True
    for u in range(T):
        ranked = O.topk_desc(sel.tile_cos[u], min(T, k + 8))
        exact &= check_topk_set(gpu_ranked[u], ranked, sel.tile_cos[u], k, f"{what} tile {u}")
    return exact


def check_token_lists(gpu_lists, L, unit, k, rows, what):
    """gpu_lists: int [S*P][S][k] per-frame patch lists of the token-wise head; rows: query
    tokens (patch tokens are checked, special ones have no list).  Each (row, frame) set must
    equal the oracle's Top-k up to the boundary band.  Returns True when all are identical."""
    exact = True
    for i in rows:
        s_i, loc = O.token_parts(L, int(i))
        if loc < L.n_special:
            continue
        a = s_i * L.P + loc - L.n_special
        cos32 = (unit @ unit[a]).astype(np.float32)
        for sv in range(L.S):
            frame = cos32[sv * L.P:(sv + 1) * L.P]
            ranked = O.topk_desc(frame, min(L.P, k + 8))
            exact &= check_topk_set(gpu_lists[a, sv], ranked, frame, k, f"{what} row {int(i)} frame {sv}")
    return exact


def selection_over_gpu_set(sel, L, h, hc, exported):
    """The oracle selection with head h's index set replaced by the one the GPU built.

    Only for a set that check_topk_set (or check_token_lists) accepted: it equals the oracle's
    own set up to keys tied within the boundary band, so it is a valid result of the selection,
    and the oracle then evaluates the exact softmax attention over it (section 4.1 of the SAF3R
    paper: each row attends exactly to its kept keys).  Where several sets are correct, this
    checks that the attention the GPU ran is the one over the set it chose."""
    s = copy.copy(sel)
    if hc.kind == O.PROBE:
        s.probe_keys = dict(sel.probe_keys)
        s.probe_keys[h] = np.sort(np.asarray(exported, dtype=np.int64))
    elif hc.kind in (O.CORR, O.HYBRID):
        s.tile_rank = np.asarray(exported, dtype=np.int64).reshape(L.T, hc.k)
    elif hc.kind == O.TOKEN:
        s.token_lists = dict(sel.token_lists)
        s.token_lists[h] = np.asarray(exported, dtype=np.int64).reshape(L.S * L.P, L.S, hc.k)
    else:
        raise ValueError(f"head kind {hc.kind} has no exported set")
    return s


class HeadSelections:
    """Per head, the selection its output rows are checked against: the oracle's own where the
    GPU's set is identical to it, else the oracle over the GPU's accepted set.  `over_gpu` names
    the heads of the second kind (printed by the tests)."""

    def __init__(self, sel):
        self.base = sel
        self.per_head = {}
        self.over_gpu = []

    def accept(self, L, h, hc, exported, exact):
        if exact:
            self.per_head[h] = self.base
        else:
            self.per_head[h] = selection_over_gpu_set(self.base, L, h, hc, exported)
            self.over_gpu.append(h)

    def __getitem__(self, h):
        return self.per_head.get(h, self.base)

    def report(self, what):
        if self.over_gpu:
            print(f"{what}: heads {self.over_gpu} resolved a boundary tie differently; their rows "
                  f"were checked over the GPU's accepted set")
