"""Pins of the CPU oracle against facts that do not come from the oracle itself:
closed forms, invariants, brute force on tiny inputs, library routines, and the
numbers printed in the SAF3R paper.  No GPU is needed."""
import math

import numpy as np
import pytest
import torch

import oracle as O
from saf3r_synth import CORR, DENSE, HYBRID, POSITION, PROBE, SCAN, TOKEN, HeadCfg, Layout

RNG = np.random.default_rng(1234)


def small_layout(S=3, g=5, H=2):
    return Layout(S=S, g=g, H=H)


# ---------------------------------------------------------------- attention

def test_single_key_returns_its_value():
    q = RNG.standard_normal(64)
    K = RNG.standard_normal((1, 64))
    V = RNG.standard_normal((1, 64))
    out = O.attention_rows(q, K, V)[0]
    assert np.array_equal(out, V[0])


def test_two_keys_closed_form_sigmoid():
    # softmax over two logits a, b is (sigmoid(a-b), sigmoid(b-a)); logits use 1/sqrt(64) = 1/8
    q = RNG.standard_normal(64)
    K = RNG.standard_normal((2, 64))
    V = RNG.standard_normal((2, 64))
    a, b = float(q @ K[0]) / 8.0, float(q @ K[1]) / 8.0
    w0 = 1.0 / (1.0 + math.exp(-(a - b)))
    expect = w0 * V[0] + (1.0 - w0) * V[1]
    np.testing.assert_allclose(O.attention_rows(q, K, V)[0], expect, rtol=0, atol=1e-13)


def test_dense_matches_torch_sdpa_fp64():
    N = 77
    Q, K, V = (RNG.standard_normal((N, 64)) for _ in range(3))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None])[0].numpy()
    np.testing.assert_allclose(O.dense_rows(Q, K, V, np.arange(N)), ref, rtol=0, atol=1e-12)


def test_sparse_matches_torch_sdpa_with_mask():
    # excluded keys behave as logit -inf: the SDPA boolean mask drops them
    N = 50
    Q, K, V = (RNG.standard_normal((N, 64)) * 2 for _ in range(3))
    keep = np.sort(RNG.choice(N, size=17, replace=False))
    mask = np.zeros((N, N), dtype=bool)
    mask[:, keep] = True
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(Q)[None], torch.from_numpy(K)[None], torch.from_numpy(V)[None],
        attn_mask=torch.from_numpy(mask)[None])[0].numpy()
    np.testing.assert_allclose(O.attention_rows(Q, K[keep], V[keep]), ref, rtol=0, atol=1e-12)


def test_softmax_rows_sum_to_one_and_identical_keys_are_uniform():
    q = RNG.standard_normal((5, 64)) * 3
    K = RNG.standard_normal((40, 64)) * 3
    w = O.attention_weights(q, K)
    assert np.all(np.abs(w.sum(axis=1) - 1.0) < 1e-12)
    Krep = np.repeat(RNG.standard_normal((1, 64)), 9, axis=0)
    V = RNG.standard_normal((9, 64))
    np.testing.assert_allclose(O.attention_rows(q, Krep, V), np.repeat(V.mean(0, keepdims=True), 5, 0),
                               rtol=0, atol=1e-13)


def test_kept_set_order_does_not_matter():
    q = RNG.standard_normal((4, 64))
    K = RNG.standard_normal((30, 64))
    V = RNG.standard_normal((30, 64))
    perm = RNG.permutation(30)
    np.testing.assert_allclose(O.attention_rows(q, K, V), O.attention_rows(q, K[perm], V[perm]),
                               rtol=0, atol=1e-12)


# ---------------------------------------------------------------- Top-K

@pytest.mark.parametrize("k", [1, 3, 7, 20])
def test_topk_equals_rank_counting_with_ties(k):
    # many duplicated scores: key j is selected iff fewer than k keys beat it,
    # where i beats j when s_i > s_j or (s_i == s_j and i < j)
    s = RNG.integers(0, 5, size=20).astype(np.float32)
    got = set(O.topk_desc(s, k).tolist())
    want = set()
    for j in range(20):
        beaten = sum(1 for i in range(20) if s[i] > s[j] or (s[i] == s[j] and i < j))
        if beaten < k:
            want.add(j)
    assert got == want
    ranked = O.topk_desc(s, k)
    assert all((s[a] > s[b]) or (s[a] == s[b] and a < b) for a, b in zip(ranked, ranked[1:]))


def test_probe_equals_column_mean_of_full_score_matrix():
    # section 4.3: ranking by the column means of QK^T/sqrt(D) equals ranking by
    # the mean-query probe.  Integer-valued Q, K make every sum exact.
    L = small_layout(S=2, g=4)
    Q = RNG.integers(-3, 4, size=(L.N, 64)).astype(np.float32)
    K = RNG.integers(-3, 4, size=(L.N, 64)).astype(np.float32)
    full = Q.astype(np.float64) @ K.astype(np.float64).T / 8.0
    colmean = full.mean(axis=0)
    patches = O.patch_tokens(L)
    for k in (1, 5, 11):
        # brute force ranking of the column means over patch keys
        order = sorted(patches.tolist(), key=lambda j: (-colmean[j], j))
        want = np.sort(np.array(order[:k]))
        got = O.probe_topk(L, O.probe_scores(O.probe_mean(Q), K), k)
        assert np.array_equal(got, want)


def test_probe_set_size_and_specials():
    L = small_layout()
    Q = RNG.standard_normal((L.N, 64)).astype(np.float32)
    K = RNG.standard_normal((L.N, 64)).astype(np.float32)
    keys = O.probe_topk(L, O.probe_scores(O.probe_mean(Q), K), 13)
    assert len(keys) == 13 and not O.is_special(L, keys).any()
    ks = O.probe_set(L, keys)
    assert len(ks) == 13 + L.n_special * L.S


# ---------------------------------------------------------------- static and stride sets

def test_position_set_closed_form_count_and_membership():
    L = small_layout(S=3, g=5)
    for i in range(L.N):
        ks = O.position_set(L, i)
        s, loc = divmod(i, L.V)
        base = L.n_special * L.S + L.P
        if loc < L.n_special:
            assert len(ks) == base
        else:
            r, c = divmod(loc - L.n_special, L.g)
            nb = (min(r + 1, L.g - 1) - max(r - 1, 0) + 1) * (min(c + 1, L.g - 1) - max(c - 1, 0) + 1)
            assert len(ks) == base + (L.S - 1) * nb
        # brute-force membership from the definition
        want = []
        for j in range(L.N):
            sj, lj = divmod(j, L.V)
            keep = lj < L.n_special or sj == 0
            if loc >= L.n_special and lj >= L.n_special:
                r, c = divmod(loc - L.n_special, L.g)
                rj, cj = divmod(lj - L.n_special, L.g)
                keep = keep or (abs(rj - r) <= 1 and abs(cj - c) <= 1)
            if keep:
                want.append(j)
        assert np.array_equal(ks, np.array(want))


def test_stride_set_closed_form():
    L = small_layout(S=3, g=5)
    for s, ph in [(1, 0), (4, 3), (7, 2), (30, 29)]:
        ks = O.stride_set(L, s, ph)
        lattice = (L.N - ph + s - 1) // s
        off = sum(1 for t in O.special_tokens(L) if t % s != ph)
        assert len(ks) == lattice + off
        assert all((j % s == ph) or (j % L.V < L.n_special) for j in ks)


def test_stride_keep_fraction_matches_paper_table6():
    rows = [l.split() for l in open("tests/golden/table6_stride_keys.txt") if l.strip() and l[0] != "#"]
    L = Layout(S=100, g=37, H=1)
    for stride, pct in rows:
        s = int(stride)
        lattice = len(O.stride_set(L, s, 0)) - sum(1 for t in O.special_tokens(L) if t % s != 0)
        assert round(100.0 * lattice / L.N, 1) == float(pct)


# ---------------------------------------------------------------- DINO tiles

def test_tile_cosines_brute_force_and_topk():
    L = small_layout(S=3, g=7)
    f = RNG.standard_normal((L.S * L.P, 16)).astype(np.float32) + 0.5
    means = O.dino_tile_means(L, f)
    # brute force: explicit loops over tokens and pairs
    for t in range(L.T):
        acc, n = np.zeros(16), 0
        for tok in range(t * 64, min(t * 64 + 64, L.N)):
            s, loc = divmod(tok, L.V)
            if loc >= L.n_special:
                row = f[s * L.P + loc - L.n_special].astype(np.float64)
                acc += row / math.sqrt(float((row * row).sum()))
                n += 1
        np.testing.assert_allclose(means[t], acc / n, rtol=0, atol=1e-14)
    cos = O.tile_cosines(means)
    for u in range(L.T):
        for v in range(L.T):
            a, b = means[u], means[v]
            want = float(a @ b) / math.sqrt(float(a @ a) * float(b @ b))
            assert abs(float(cos[u, v]) - want) <= 1e-6
    rank = O.tile_topk(cos, L.T)
    for u in range(L.T):
        assert sorted(rank[u].tolist()) == list(range(L.T))
        assert rank[u][0] == u or cos[u, rank[u][0]] >= cos[u, u]


def test_corr_set_dedups_specials():
    L = small_layout(S=3, g=7)
    tiles = [0, 2]
    ks = O.corr_set(L, tiles)
    inside = sum(1 for v in tiles for t in O.tile_tokens(L, v) if t % L.V < L.n_special)
    assert len(ks) == sum(len(O.tile_tokens(L, v)) for v in tiles) + L.n_special * L.S - inside
    assert len(set(ks.tolist())) == len(ks)


# ---------------------------------------------------------------- reductions to dense

def test_full_budgets_reduce_to_dense():
    L = small_layout(S=2, g=6)
    Q, K, V = (RNG.standard_normal((1, L.N, 64)).astype(np.float32) for _ in range(3))
    dino = RNG.standard_normal((L.S * L.P, 8)).astype(np.float32)
    rows = np.arange(L.N)
    dense = O.dense_rows(Q[0], K[0], V[0], rows)
    for hc in [HeadCfg(PROBE, k=L.S * L.P), HeadCfg(SCAN, stride=1, phase=0), HeadCfg(CORR, k=L.T),
               HeadCfg(DENSE), HeadCfg(HYBRID, k=1, stride=1, phase=0), HeadCfg(HYBRID, k=L.T, stride=7, phase=2)]:
        sel = O.select(L, [hc], Q, K, dino)
        out = O.sparse_rows(L, hc, sel, 0, Q[0], K[0], V[0], rows)
        np.testing.assert_allclose(out, dense, rtol=0, atol=1e-12)
        assert O.nmse(dense, out) < 1e-24
    L1 = Layout(S=1, g=6, H=1)
    Q1, K1, V1 = (RNG.standard_normal((L1.N, 64)) for _ in range(3))
    sel = O.Selection()
    out = O.sparse_rows(L1, HeadCfg(POSITION), sel, 0, Q1, K1, V1, np.arange(L1.N))
    np.testing.assert_allclose(out, O.dense_rows(Q1, K1, V1, np.arange(L1.N)), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- NMSE and the profile rule

def test_nmse_closed_forms():
    a = RNG.standard_normal((10, 64))
    assert O.nmse(a, a) == 0.0
    for alpha in (0.0, 0.5, 1.5):
        assert abs(O.nmse(a, alpha * a) - (1 - alpha) ** 2) < 1e-14


def test_choose_config_rule():
    # cheapest qualifying candidate; ties in cost to the lower index
    assert O.choose_config([0.5, 0.005, 0.009, 0.001], [10, 40, 30, 30], 1e-2) == 2
    # nothing qualifies -> least NMSE, ties to the lower index
    assert O.choose_config([0.5, 0.2, 0.2], [1, 2, 3], 1e-2) == 1
    assert O.choose_config([0.01, 0.02], [5, 1], 1e-2) == 0


def test_kept_pairs_and_omega():
    L = small_layout(S=2, g=4)
    sel = O.Selection()
    pairs = O.kept_pairs(L, HeadCfg(SCAN, stride=3, phase=1), sel, 0)
    assert pairs == L.N * len(O.stride_set(L, 3, 1))
    assert O.omega(L, pairs) == 256 * pairs


def test_baseline_stride():
    # keeping one key in s is sparsity 1 - 1/s; the smallest s reaching sigma
    assert O.baseline_stride(0.85) == 7        # 1 - 1/7 = 0.857 >= 0.85 > 1 - 1/6
    assert O.baseline_stride(0.75) == 4
    assert O.baseline_stride(0.0) == 1
    for sigma in np.linspace(0.0, 0.95, 40):
        s = O.baseline_stride(float(sigma))
        assert 1 - 1 / s >= sigma - 1e-12 and (s == 1 or 1 - 1 / (s - 1) < sigma)


def _eq2_brute(E, W, base):
    """eq. 2 restated as a constrained argmin: least error among the candidates that cost no
    more than the baseline; ties to the baseline, then to the lower index."""
    H, C = E.shape
    out = []
    for h in range(H):
        feas = [c for c in range(C) if W[h, c] <= W[h, base]]
        out.append(min(feas, key=lambda c: (E[h, c], 0 if c == base else 1, c)))
    return out


def test_choose_eq2_rule():
    # head 0: candidate 1 is cheaper and better; 2 is better still but costs more than the baseline
    # head 1: nothing under the baseline cost beats it -> the baseline stays
    # head 2: equal error to the baseline -> the baseline stays
    E = np.array([[0.5, 0.4, 0.1, 0.45], [0.2, 0.3, 0.25, 0.1], [0.3, 0.3, 0.3, 0.3]])
    W = np.array([[100, 90, 120, 80], [100, 60, 100, 101], [100, 50, 50, 50]])
    assert O.choose_eq2([E], [W], 0) == [1, 0, 0]
    # averaging over inputs: the second input flips head 0's order of 1 and 3
    E2 = E.copy()
    E2[0] = [0.5, 0.6, 0.1, 0.2]
    assert O.choose_eq2([E, E2], [W, W], 0) == [3, 0, 0]


def test_choose_eq2_equals_constrained_argmin():
    rng = np.random.default_rng(7)
    for _ in range(200):
        H, C = int(rng.integers(1, 5)), int(rng.integers(1, 8))
        n_in = int(rng.integers(1, 4))
        Es = rng.choice([0.1, 0.2, 0.3, 0.4], size=(n_in, H, C))    # coarse values: many ties
        Ws = rng.integers(1, 5, size=(n_in, H, C)) * 10
        base = int(rng.integers(0, C))
        got = O.choose_eq2(Es, Ws, base)
        assert got == _eq2_brute(Es.mean(axis=0), Ws.mean(axis=0), base)
        E, W = Es.mean(axis=0), Ws.mean(axis=0)
        for h, c in enumerate(got):
            assert W[h, c] <= W[h, base] and E[h, c] <= E[h, base]


def test_hybrid_set_counts_and_pieces():
    """The hybrid set is the tile set united with the stride set: its size by inclusion-exclusion
    over the tokens of the kept tiles, and each piece alone when the other is empty or full."""
    L = small_layout(S=3, g=7)   # V = 54, N = 162, three tiles (the last one partial)
    dino = RNG.standard_normal((L.S * L.P, 8)).astype(np.float32)
    Q = K = RNG.standard_normal((1, L.N, 64)).astype(np.float32)
    for k, stride, phase in [(1, 5, 3), (2, 9, 0), (1, 64, 63), (3, 2, 1)]:
        hc = HeadCfg(HYBRID, k=k, stride=stride, phase=phase)
        sel = O.select(L, [hc], Q, K, dino)
        lattice = set(range(phase, L.N, stride))
        specials = {s * L.V + i for s in range(L.S) for i in range(L.n_special)}
        for i in (0, 60, L.N - 1):
            tiles = sel.tile_rank[i // 64, :k]
            tile_tokens = {t for v in tiles for t in range(64 * int(v), min(L.N, 64 * int(v) + 64))}
            patch_in_tiles = tile_tokens - specials
            want = len(lattice | specials) + len(patch_in_tiles - lattice)
            got = O.key_set(L, hc, sel, 0, i)
            assert len(got) == want and len(set(got.tolist())) == want
            assert set(got.tolist()) == lattice | specials | patch_in_tiles
        assert O.kept_pairs(L, hc, sel, 0) == sum(O.kept_count(L, hc, sel, 0, i) for i in range(L.N))


def test_anchor_frame_only_static_set():
    L = small_layout(S=3, g=4)
    specials = {s * L.V + i for s in range(L.S) for i in range(L.n_special)}
    want = specials | set(range(L.V))
    for i in range(L.N):
        assert set(O.position_set(L, i, radius=-1).tolist()) == want


def test_token_topk_brute_force_and_counts():
    """Token-wise per-frame Top-K against a brute-force sort of explicit cosines, the own token
    first in its own frame, k = P reducing to every key, and the closed-form pair count."""
    L = small_layout(S=3, g=4)   # P = 16 patches per frame
    dino = RNG.standard_normal((L.S * L.P, 12)).astype(np.float32)
    unit = O.unit_features(dino)
    for i in [L.n_special, L.V + L.n_special + 7, L.N - 1]:
        s_i, loc = O.token_parts(L, i)
        a = s_i * L.P + loc - L.n_special
        for k in (1, 3, L.P):
            got = O.token_topk_row(L, unit, i, k)
            for sv in range(L.S):
                cos = [float(np.float32(np.dot(dino[a], dino[sv * L.P + p]) /
                                        (np.linalg.norm(dino[a].astype(np.float64)) *
                                         np.linalg.norm(dino[sv * L.P + p].astype(np.float64)))))
                       for p in range(L.P)]
                want = sorted(range(L.P), key=lambda p: (-cos[p], p))[:k]
                assert got[sv].tolist() == want
            assert got[s_i][0] == a - s_i * L.P  # a token is most similar to itself
    hc = HeadCfg(TOKEN, k=L.P)
    sel = O.select(L, [hc], None, None, dino)
    for i in (0, L.n_special, L.N - 1):
        assert O.key_set(L, hc, sel, 0, i).tolist() == list(range(L.N))
    hc = HeadCfg(TOKEN, k=2)
    sel = O.select(L, [hc], None, None, dino)
    assert O.kept_pairs(L, hc, sel, 0) == sum(len(O.key_set(L, hc, sel, 0, i)) for i in range(L.N))


# ---------------------------------------------------------------- precision of the selection
def test_selection_stable_under_fp32_accumulation():
    """Every reduction of the selection run in fp32 instead of fp64 gives the same index sets,
    up to keys whose fp64 score lies within the acceptance band (1e-5 relative) of the k-th
    score: the probe, tile and token Top-K sets do not hinge on the accumulation precision, so a
    GPU that forms scores in fp32 and recomputes only near-ties exactly selects the same keys."""
    from parity_util import check_token_lists, check_topk_set
    from saf3r_synth import Scene, Workload, bf16_to_f32, qkv
    L = Layout(S=8, g=16, H=4)
    heads = [HeadCfg(PROBE, k=300), HeadCfg(CORR, k=6), HeadCfg(TOKEN, k=12), HeadCfg(SCAN, stride=4, phase=1)]
    wl = Workload("fp32-accumulation", L, M=256, delta=11, D=128, heads=heads, seed=9)
    scene = Scene(wl)
    Q, K, _ = (bf16_to_f32(t) for t in qkv(scene, 0))
    dino = scene.dino()
    s64 = O.select(L, heads, Q, K, dino)
    s32 = O.select(L, heads, Q, K, dino, accum=np.float32)
    assert s32.unit.dtype == np.float32 and s32.tile_cos is not None
    sc = s64.probe_scores[0]
    check_topk_set(s32.probe_keys[0], O.topk_desc(sc, 308, O.patch_tokens(L)), sc, 300, "probe fp32")
    for u in range(L.T):
        check_topk_set(s32.tile_rank[u, :6], O.topk_desc(s64.tile_cos[u], 14), s64.tile_cos[u], 6, f"tile {u} fp32")
    lists = np.zeros((L.S * L.P, L.S, 12), dtype=np.int64)
    rows = [i for i in range(L.N) if O.token_parts(L, i)[1] >= L.n_special]
    for i in rows:
        s_i, loc = O.token_parts(L, i)
        lists[s_i * L.P + loc - L.n_special] = O.token_topk_row(L, s32.unit, i, 12)
    check_token_lists(lists, L, s64.unit, 12, rows, "token fp32")


# ---------------------------------------------------------------- row batching of the oracle

@pytest.mark.parametrize("hc", [HeadCfg(POSITION), HeadCfg(POSITION, radius=0), HeadCfg(POSITION, radius=2),
                                HeadCfg(POSITION, radius=-1), HeadCfg(PROBE, k=30), HeadCfg(CORR, k=2),
                                HeadCfg(HYBRID, k=2, stride=5, phase=3), HeadCfg(SCAN, stride=4, phase=1),
                                HeadCfg(DENSE), HeadCfg(TOKEN, k=3)])
def test_sparse_rows_batching_equals_one_row_at_a_time(hc):
    """sparse_rows evaluates rows in batches of equal key sets; each output row must equal the
    plain attention of that row over its own key set, taken one row at a time (rows given in a
    shuffled order, three views so that rows of the same grid cell and tile sit in different views)."""
    L = Layout(S=3, g=6, H=1)
    rng = np.random.default_rng(77)
    Q, K, V = (rng.standard_normal((1, L.N, 64)) for _ in range(3))
    dino = rng.standard_normal((L.S * L.P, L.dino_dim)).astype(np.float32)
    sel = O.select(L, [hc], Q, K, dino)
    rows = rng.permutation(L.N)
    got = O.sparse_rows(L, hc, sel, 0, Q[0], K[0], V[0], rows)
    for n, i in enumerate(rows):
        keys = O.key_set(L, hc, sel, 0, int(i))
        want = O.attention_rows(Q[0][i], K[0][keys], V[0][keys])[0]
        np.testing.assert_allclose(got[n], want, rtol=0, atol=1e-12, err_msg=f"row {i}")


def test_given_token_lists_replace_the_ranking():
    """A token-wise head evaluated over given per-frame lists: the oracle's own lists give the
    same sets as its ranking, and a list that swaps one key changes exactly that row's set."""
    L = Layout(S=3, g=5, H=1)
    rng = np.random.default_rng(78)
    dino = rng.standard_normal((L.S * L.P, L.dino_dim)).astype(np.float32)
    hc = HeadCfg(TOKEN, k=2)
    sel = O.select(L, [hc], None, None, dino)
    lists = np.stack([O.token_topk_row(L, sel.unit, L.n_special + p % L.P + (p // L.P) * L.V, 2)
                      for p in range(L.S * L.P)])
    given = O.Selection()
    given.unit = sel.unit
    given.token_lists = {0: lists}
    for i in range(L.N):
        assert np.array_equal(O.key_set(L, hc, sel, 0, i), O.key_set(L, hc, given, 0, i))
    swapped = lists.copy()
    i = 2 * L.V + L.n_special + 7  # view 2, patch 7
    a = 2 * L.P + 7
    old = swapped[a, 1, 1]
    new = next(p for p in range(L.P) if p not in swapped[a, 1])
    swapped[a, 1, 1] = new
    given.token_lists = {0: swapped}
    diff = set(O.key_set(L, hc, sel, 0, i).tolist()) ^ set(O.key_set(L, hc, given, 0, i).tolist())
    assert diff == {1 * L.V + L.n_special + old, 1 * L.V + L.n_special + new}
    assert np.array_equal(O.key_set(L, hc, sel, 0, i + 1), O.key_set(L, hc, given, 0, i + 1))


def test_nmse_sample_estimate_within_its_standard_error():
    """eq. 1's NMSE on all query rows against its row-sample estimate.  On a layer small enough for
    every row: (1) the all-row table equals sum_i |O_f,i - O_s,i|^2 / sum_i |O_f,i|^2 with the dense
    rows from torch's fp64 SDPA; (2) a 300-row sample's value (a ratio estimate) lies within 6
    standard errors of it, the error estimated from the per-row terms, for every head and
    candidate.  This pins the sampled form used at full size by its sampling distribution."""
    L = Layout(S=4, g=20, H=2)
    rng = np.random.default_rng(99)
    Q, K, V = (rng.standard_normal((L.H, L.N, 64)) for _ in range(3))
    dino = rng.standard_normal((L.S * L.P, L.dino_dim)).astype(np.float32)
    cands = [HeadCfg(PROBE, k=150), HeadCfg(SCAN, stride=4), HeadCfg(POSITION), HeadCfg(CORR, k=3)]
    every = [np.arange(L.N)] * L.H
    table = O.nmse_table_sampled(L, cands, Q, K, V, dino, every)
    n = 300
    sample = [np.sort(rng.choice(L.N, size=n, replace=False)) for _ in range(L.H)]
    est = O.nmse_table_sampled(L, cands, Q, K, V, dino, sample)
    for h in range(L.H):
        q = torch.from_numpy(Q[h])[None, None]
        dense = torch.nn.functional.scaled_dot_product_attention(
            q, torch.from_numpy(K[h])[None, None], torch.from_numpy(V[h])[None, None], scale=0.125)[0, 0].numpy()
        for c, cand in enumerate(cands):
            hc = O.apply_candidate(cand, h)
            heads = [O.apply_candidate(cand, x) for x in range(L.H)]
            sel = O.select(L, heads, Q, K, dino)
            sparse = O.sparse_rows(L, hc, sel, h, Q[h], K[h], V[h], np.arange(L.N))
            a = np.sum((dense - sparse) ** 2, axis=1)
            b = np.sum(dense ** 2, axis=1)
            R = a.sum() / b.sum()
            assert abs(table[h, c] - R) <= 1e-9 * max(R, 1e-12), (h, c, table[h, c], R)
            se = math.sqrt((1.0 - n / L.N) * np.var(a - R * b) / n) / b.mean()
            assert abs(est[h, c] - R) <= 6.0 * se + 1e-12, (h, c, est[h, c], R, se)
