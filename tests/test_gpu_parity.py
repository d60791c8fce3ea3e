"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Index sets must match exactly up to the boundary band;
outputs within max-abs 1e-2 and rel-L2 5e-3."""
import numpy as np
import pytest

import oracle as O
from saf3r_synth import (CORR, DENSE, HYBRID, POSITION, PROBE, SCAN, TOKEN, WORKLOADS, HeadCfg, Layout, Scene,
                         Workload, bf16_to_f32, qkv, sample_rows)
from parity_util import HeadSelections, check_probe, check_tiles, check_token_lists, compare_outputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _hw():
    import head_wise_dynamic_b200 as hw
    return hw


class Case:
    """Inputs of one layer on the GPU plus their exact fp32 copies for the oracle."""

    def __init__(self, wl: Workload, layer: int = 0, seed=None):
        self.wl = wl
        self.L = wl.layout
        self.scene = Scene(wl, seed)
        self.q, self.k, self.v = qkv(self.scene, layer, device="cuda")
        self.dino = torch.from_numpy(self.scene.dino()).cuda()
        self.Q, self.K, self.V = (bf16_to_f32(t) for t in (self.q, self.k, self.v))


def run_gpu(case, heads, out_fp32=True):
    hw = _hw()
    att = hw.SparseGlobalAttention(case.L, heads, out_dtype=torch.float32 if out_fp32 else torch.bfloat16)
    att.select(case.q, case.k, case.dino)
    att.out.fill_(float("nan"))  # every row must be written by the kernel
    out = att(case.q, case.k, case.v)
    torch.cuda.synchronize()
    hw.saf3r_check()
    return att, out


def oracle_select(case, heads):
    return O.select(case.L, heads, case.Q, case.K, case.dino.cpu().numpy())


def check_selection(case, heads, att, sel):
    """Every exported index set against the oracle's (exact up to the boundary band); returns the
    per-head selections the output rows are checked against (HeadSelections)."""
    hw = _hw()
    sels = HeadSelections(sel)
    for h, hc in enumerate(heads):
        if hc.kind == PROBE:
            keys = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h)
            sels.accept(case.L, h, hc, keys, check_probe(keys, case.L, sel, h, hc.k, f"probe head {h}"))
        elif hc.kind in (CORR, HYBRID):
            ranked = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).reshape(case.L.T, hc.k)
            sels.accept(case.L, h, hc, ranked, check_tiles(ranked, sel, hc.k, f"tile head {h}"))
    return sels


def check_rows(case, heads, sels, out, rows_per_head):
    """Output rows of every head against the oracle over that head's (validated) set: no head is
    skipped, also where a boundary tie made the GPU's set differ from the oracle's."""
    out = out.float().cpu().numpy()
    for h, hc in enumerate(heads):
        rows = rows_per_head(h)
        ref = O.sparse_rows(case.L, hc, sels[h], h, case.Q[h], case.K[h], case.V[h], rows)
        compare_outputs(out[h][rows], ref, f"head {h} ({hc.kind})")
    sels.report(case.wl.name)


@pytest.fixture(scope="module")
def tiny():
    return Case(WORKLOADS["tiny"])


@pytest.mark.parametrize("out_fp32", [True, False])
def test_tiny_all_rows(tiny, out_fp32):
    heads = tiny.wl.heads
    att, out = run_gpu(tiny, heads, out_fp32)
    sel = oracle_select(tiny, heads)
    sels = check_selection(tiny, heads, att, sel)
    check_rows(tiny, heads, sels, out, lambda h: np.arange(tiny.L.N))


def test_tiny_dense(tiny):
    hw = _hw()
    L = hw.layout_of(tiny.L)
    out = torch.empty((tiny.L.H, tiny.L.N, 64), dtype=torch.float32, device="cuda")
    ws = torch.empty(hw.saf3r_workspace_bytes(L, None, hw.OP_DENSE), dtype=torch.uint8, device="cuda")
    hw.saf3r_dense_attn(L, tiny.q, tiny.k, tiny.v, out, ws)
    torch.cuda.synchronize()
    hw.saf3r_check()
    o = out.cpu().numpy()
    for h in range(tiny.L.H):
        compare_outputs(o[h], O.dense_rows(tiny.Q[h], tiny.K[h], tiny.V[h], np.arange(tiny.L.N)), f"dense {h}")


def test_deterministic(tiny):
    heads = tiny.wl.heads
    _, a = run_gpu(tiny, heads)
    _, b = run_gpu(tiny, heads)
    assert torch.equal(a, b)


def _custom(S, g, heads, seed=7, M=256, D=128, ns=5):
    L = Layout(S=S, g=g, H=len(heads), n_special=ns)
    return Workload("custom", L, M=M, delta=11, D=D, heads=heads, seed=seed)


EDGE = {
    # N = 258: ragged last 256-row item, last tile of 2 tokens
    "ragged": _custom(3, 9, [HeadCfg(POSITION), HeadCfg(PROBE, k=40), HeadCfg(CORR, k=2),
                             HeadCfg(SCAN, stride=5, phase=4)]),
    # one view: every head sees all keys of view 0
    "one_view": _custom(1, 12, [HeadCfg(POSITION), HeadCfg(PROBE, k=144), HeadCfg(CORR, k=3),
                                HeadCfg(SCAN, stride=1, phase=0)]),
    # full budgets reduce to dense attention; radius 0 and 2
    "full_budgets": _custom(2, 10, [HeadCfg(PROBE, k=200), HeadCfg(CORR, k=4), HeadCfg(SCAN, stride=1),
                                    HeadCfg(DENSE), HeadCfg(POSITION, radius=0), HeadCfg(POSITION, radius=2)]),
    # many views per item (S = 5 < 256): several cells per work item; a 3-head layout
    "many_cells": _custom(5, 11, [HeadCfg(POSITION), HeadCfg(SCAN, stride=3, phase=1), HeadCfg(CORR, k=5),
                                  HeadCfg(POSITION, radius=-1)]),
    # larger than one 128-key block per run; big probe K spanning many blocks
    "multi_block": _custom(6, 16, [HeadCfg(PROBE, k=700), HeadCfg(POSITION), HeadCfg(SCAN, stride=2, phase=1),
                                   HeadCfg(CORR, k=9)]),
    # tiles united with a stride lattice: ragged layout; a lattice of one key per tile; stride 1
    # (every key); a plain correspondence head with the same budget sharing the tile lists
    "hybrid_ragged": _custom(3, 9, [HeadCfg(HYBRID, k=2, stride=5, phase=4), HeadCfg(HYBRID, k=1, stride=64, phase=63),
                                    HeadCfg(HYBRID, k=3, stride=1, phase=0), HeadCfg(CORR, k=2)]),
    # several blocks per run, two hybrid heads whose derived runs differ in length
    "hybrid_multi": _custom(6, 16, [HeadCfg(HYBRID, k=9, stride=7, phase=3), HeadCfg(HYBRID, k=4, stride=16, phase=0),
                                    HeadCfg(SCAN, stride=7, phase=3), HeadCfg(CORR, k=9)]),
}


@pytest.mark.parametrize("name", list(EDGE))
def test_edge_cases_all_rows(name):
    case = Case(EDGE[name])
    heads = case.wl.heads
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    sels = check_selection(case, heads, att, sel)
    check_rows(case, heads, sels, out, lambda h: np.arange(case.L.N))


def test_cache_mismatch_is_reported_and_out_untouched(tiny):
    hw = _hw()
    heads = tiny.wl.heads
    att, _ = run_gpu(tiny, heads)
    other = list(heads)
    other[1] = HeadCfg(PROBE, k=64)  # different probe budget: the header hash differs
    cfg2 = hw.cfg_array(other)
    ws = torch.empty(hw.saf3r_workspace_bytes(att.layout, cfg2, hw.OP_SPARSE), dtype=torch.uint8, device="cuda")
    out = torch.full((tiny.L.H, tiny.L.N, 64), 7.0, dtype=torch.float32, device="cuda")
    hw.saf3r_sparse_attn(att.layout, cfg2, att.cache, tiny.q, tiny.k, tiny.v, out, ws)
    with pytest.raises(hw.Saf3rError) as e:
        hw.saf3r_check()
    assert e.value.status == hw.ERR_INVALID
    assert bool((out == 7.0).all())
    hw.saf3r_check()  # the error word was cleared


@pytest.fixture(scope="module")
def s32():
    return Case(WORKLOADS["s32"])


def test_s32_selection_and_sampled_rows(s32):
    heads = s32.wl.heads
    att, out = run_gpu(s32, heads, out_fp32=False)
    sel = oracle_select(s32, heads)
    sels = check_selection(s32, heads, att, sel)
    check_rows(s32, heads, sels, out, lambda h: sample_rows(s32.wl, h, 512))


def test_s32_hybrid_heads_sampled_rows_and_pairs(s32):
    """Tile Top-32 united with stride-20 lattices (phase = head mod 20) on the S=32 layer."""
    hw = _hw()
    heads = [HeadCfg(HYBRID, k=32, stride=20, phase=h % 20) for h in range(s32.L.H)]
    att, out = run_gpu(s32, heads, out_fp32=False)
    sel = oracle_select(s32, heads)
    sels = check_selection(s32, heads, att, sel)
    check_rows(s32, heads, sels, out, lambda h: sample_rows(s32.wl, h, 256))
    pairs = hw.saf3r_kept_pairs(att.layout, att.cfg, att.cache)
    for h in (0, 7):
        assert int(pairs[h]) == O.kept_pairs(s32.L, heads[h], sels[h], h)


# ---------------------------------------------------------------- forced ties of the probe and tile Top-K

@pytest.mark.parametrize("n_rows", [3, 17])
def test_probe_ties_go_to_the_lower_index(n_rows):
    """Every patch key of the probe heads takes one of n_rows distinct K rows, so the probe scores
    tie in groups and the k-th score falls inside a tie group (k = 1 takes one of a group).  Ties
    go to the lower token index on both sides (section 4.3's Top-K, read with that tie rule), so
    the sets must be identical, not merely equal up to the boundary band."""
    case = Case(_custom(4, 12, [HeadCfg(PROBE, k=100), HeadCfg(PROBE, k=37), HeadCfg(PROBE, k=1),
                                HeadCfg(SCAN, stride=3, phase=1)], seed=70 + n_rows))
    L = case.L
    rng = np.random.default_rng(700 + n_rows)
    patch = O.patch_tokens(L)
    tmpl = patch[rng.choice(len(patch), size=n_rows, replace=False)]
    src = np.arange(L.N)
    src[patch] = tmpl[rng.integers(0, n_rows, size=len(patch))]
    src_t = torch.from_numpy(src).cuda()
    for h in range(3):
        case.k[h] = case.k[h][src_t]
    case.K = bf16_to_f32(case.k)
    heads = case.wl.heads
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    for h in range(3):  # the ties really are at the boundary
        sc = sel.probe_scores[h][patch]
        kth = np.sort(sc)[::-1][heads[h].k - 1]
        assert np.count_nonzero(sc == kth) > 1
    sels = check_selection(case, heads, att, sel)
    assert not sels.over_gpu, f"probe heads {sels.over_gpu} broke a tie differently from the oracle"
    check_rows(case, heads, sels, out, lambda h: np.arange(L.N))


@pytest.mark.parametrize("n_rows", [2, 3])
def test_probe_ties_span_key_chunks(n_rows):
    """As above on a layer of 12,840 keys, so a tie group is spread over every 4,096-key chunk
    of the multi-block radix select: the equal keys taken must be the lowest-index ones across
    chunks, not within each chunk.  Budgets cut through a tie group (k = 5000 and 4300 with 2 or
    3 groups of ~4,300-6,400 keys)."""
    heads = [HeadCfg(PROBE, k=5000), HeadCfg(PROBE, k=4300), HeadCfg(PROBE, k=1), HeadCfg(SCAN, stride=4, phase=3)]
    case = Case(_custom(8, 40, heads, seed=90 + n_rows))
    L = case.L
    assert L.N > 3 * 4096
    rng = np.random.default_rng(900 + n_rows)
    patch = O.patch_tokens(L)
    tmpl = patch[rng.choice(len(patch), size=n_rows, replace=False)]
    src = np.arange(L.N)
    src[patch] = tmpl[rng.integers(0, n_rows, size=len(patch))]
    src_t = torch.from_numpy(src).cuda()
    for h in range(3):
        case.k[h] = case.k[h][src_t]
    case.K = bf16_to_f32(case.k)
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    for h in range(3):
        sc = sel.probe_scores[h][patch]
        kth = np.sort(sc)[::-1][heads[h].k - 1]
        tied = patch[sc == kth]
        assert len(tied) > 1 and tied.min() < 4096 and tied.max() >= 3 * 4096
    sels = check_selection(case, heads, att, sel)
    assert not sels.over_gpu, f"probe heads {sels.over_gpu} broke a tie differently from the oracle"
    rows = np.sort(rng.choice(L.N, size=384, replace=False))
    check_rows(case, heads, sels, out, lambda h: rows)


@pytest.mark.parametrize("period", [2, 3])
def test_tile_ties_go_to_the_lower_index(period):
    """Views s and s + period get the same DINO features on a layout whose views are exactly two
    64-token tiles (11x11 patches + 7 special tokens = 128 tokens), so the tiles of those views
    have identical means and every query tile sees exact cosine ties, its own tile among them.
    Budgets cut through the tie groups; ties go to the lower tile index on both sides, so the
    ranked lists of the correspondence and hybrid heads must be identical to the oracle's."""
    heads = [HeadCfg(CORR, k=2), HeadCfg(CORR, k=4), HeadCfg(HYBRID, k=5, stride=7, phase=2),
             HeadCfg(HYBRID, k=1, stride=16, phase=0)]
    case = Case(_custom(6, 11, heads, seed=80 + period, ns=7))
    L = case.L
    assert L.V == 128 and L.T == 2 * L.S
    base = case.dino.cpu().numpy()[:period * L.P].reshape(period, L.P, L.dino_dim)
    case.dino = torch.from_numpy(np.ascontiguousarray(
        np.concatenate([base[s % period] for s in range(L.S)], axis=0))).cuda()
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    for u in range(L.T):  # each tile's copies tie with it exactly
        assert np.count_nonzero(sel.tile_cos[u] == sel.tile_cos[u, u]) == L.S // period
    sels = check_selection(case, heads, att, sel)
    assert not sels.over_gpu, f"tile heads {sels.over_gpu} broke a tie differently from the oracle"
    check_rows(case, heads, sels, out, lambda h: np.arange(L.N))


def test_tile_rank_with_more_candidates_than_its_list():
    """Every patch gets the same DINO feature on a 160-view layout of two-tile views (T = 320), so
    every tile mean is the same vector and each query tile's row holds T candidates within the
    tensor-core bound of its k-th cosine: more than the ranking kernel's list of 256, so the row
    is recomputed in place (its second path).  The oracle's means are exactly equal (all ties, the
    lowest tile indices win); the GPU's fp32 means may differ in the last bits, so its lists are
    accepted within the boundary band and the outputs compared over them."""
    heads = [HeadCfg(CORR, k=64), HeadCfg(CORR, k=300), HeadCfg(HYBRID, k=7, stride=9, phase=4),
             HeadCfg(POSITION)]
    case = Case(_custom(160, 11, heads, seed=85, ns=7))
    L = case.L
    assert L.V == 128 and L.T == 320
    case.dino = case.dino[:1].expand(L.S * L.P, L.dino_dim).contiguous()
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    assert np.all(sel.tile_cos == sel.tile_cos[0, 0])  # every cosine ties in the oracle
    sels = check_selection(case, heads, att, sel)
    rows = np.sort(np.random.default_rng(850).choice(L.N, size=256, replace=False))
    check_rows(case, heads, sels, out, lambda h: rows)


# ---------------------------------------------------------------- token-wise per-frame DINO Top-K

TOKEN_CASES = {
    # ragged layout; k = P keeps every key; k = 1; a main-kernel head beside them
    "token_ragged": _custom(3, 9, [HeadCfg(TOKEN, k=3), HeadCfg(TOKEN, k=81), HeadCfg(TOKEN, k=1),
                                   HeadCfg(SCAN, stride=5, phase=4)]),
    # token-wise heads mixed with the other kinds in one call
    "token_mixed": _custom(4, 16, [HeadCfg(TOKEN, k=16), HeadCfg(CORR, k=4), HeadCfg(TOKEN, k=5),
                                   HeadCfg(POSITION)], D=256),
    # no special tokens: every item's keys are its union alone
    "token_no_specials": _custom(3, 10, [HeadCfg(TOKEN, k=6), HeadCfg(SCAN, stride=3, phase=1),
                                         HeadCfg(TOKEN, k=2), HeadCfg(PROBE, k=30)], ns=0),
    # one view: the query order has no second frame; k = P keeps the whole view
    "token_one_view": _custom(1, 12, [HeadCfg(TOKEN, k=7), HeadCfg(TOKEN, k=144), HeadCfg(CORR, k=2),
                                      HeadCfg(POSITION)]),
}


@pytest.mark.parametrize("which", ["probe", "tile", "token_order", "token_union"])
def test_out_of_range_cached_index_is_reported(tiny, which):
    """A cached index that points outside the layer is range-checked where it is consumed: the
    call records SAF3R_ERR_INDEX, reads nothing out of range, and the next check finds the error
    word cleared.  Planted values: a probe key past N, a ranked tile past T, a token-wise patch
    query past S*P in the cached query order, a token past N in an item's union.  The cache
    header's hash covers the layout and the configuration, not the lists, so the planted value
    gets past the cache check."""
    hw = _hw()
    case = tiny if which in ("probe", "tile") else Case(TOKEN_CASES["token_mixed"])
    heads = case.wl.heads
    L = case.L
    att, _ = run_gpu(case, heads)
    words = att.cache.view(torch.int32).cpu().numpy().copy()

    def find(lst):
        starts = [i for i in np.flatnonzero(words[:len(words) - len(lst) + 1] == lst[0])
                  if np.array_equal(words[i:i + len(lst)], lst)]
        assert len(starts) == 1, "the exported list is not one contiguous run of the cache"
        return starts[0]

    if which in ("probe", "tile"):
        h = 1 if which == "probe" else 2
        assert heads[h].kind == (PROBE if which == "probe" else CORR)
        lst = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).ravel().astype(np.int32)
        words[find(lst) + len(lst) // 2] = L.N + 7 if which == "probe" else L.T + 5
    else:
        # head 0 has the widest per-frame budget, so its lists are the cached block itself; the
        # query order follows it (64-word aligned), then the first group's union lengths and unions
        assert heads[0].kind == TOKEN and heads[0].k == max(hc.k for hc in heads if hc.kind == TOKEN)
        lst = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, 0).ravel().astype(np.int32)
        R = L.S * L.P
        perm_at = (find(lst) + len(lst) + 63) // 64 * 64
        assert np.array_equal(np.sort(words[perm_at:perm_at + R]), np.arange(R))  # a permutation
        if which == "token_order":
            words[perm_at + R // 2] = R + 3
        else:
            items = (R + 255) // 256
            tn_at = (perm_at + R + 63) // 64 * 64
            tu_at = (tn_at + items + 63) // 64 * 64
            U0 = int(words[tn_at])
            first = words[tu_at:tu_at + U0]
            assert 0 < U0 and np.all(np.diff(first) > 0) and first[-1] < L.N  # item 0's union, ascending
            words[tu_at + U0 // 2] = L.N + 11
    att.cache.copy_(torch.from_numpy(words).view(torch.uint8).to(att.cache.device))
    att(case.q, case.k, case.v)
    with pytest.raises(hw.Saf3rError) as e:
        hw.saf3r_check()
    assert e.value.status == hw.ERR_INDEX
    hw.saf3r_check()  # the error word was cleared

def test_token_unions_are_exactly_their_rows_keys():
    """The token-wise structures of a built cache, checked exactly on the host against the cached
    per-frame lists: the patch query order is a permutation of the S*P patch queries; for every
    budget k (one group per distinct k, in head order) and every 256 queries of the order, the union
    is the ascending set of tokens those queries keep (their first k list entries of every frame),
    and query r's mask bit for union entry e is set exactly when r keeps that token (rows past the
    last query keep nothing).  Placement: after the lists, each region starts on a 64-word boundary:
    the order, then per group the union lengths, the unions (ucap = S*min(256k, P) rounded up to 64
    entries per item) and the masks ([ucap/64][256] 64-bit words per item)."""
    hw = _hw()
    case = Case(TOKEN_CASES["token_mixed"])
    heads = case.wl.heads
    L = case.L
    att, _ = run_gpu(case, heads)
    words = att.cache.view(torch.int32).cpu().numpy()
    ks = []
    for hc in heads:
        if hc.kind == TOKEN and hc.k not in ks:
            ks.append(hc.k)
    kmax = max(ks)
    h0 = [i for i, hc in enumerate(heads) if hc.kind == TOKEN and hc.k == kmax][0]
    lst = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h0).ravel().astype(np.int32)
    at = [i for i in np.flatnonzero(words[:len(words) - len(lst) + 1] == lst[0])
          if np.array_equal(words[i:i + len(lst)], lst)]
    assert len(at) == 1
    R, S, P, V, ns = L.S * L.P, L.S, L.P, L.V, L.n_special
    lists = lst.reshape(R, S, kmax)
    al = lambda x: (x + 63) // 64 * 64
    perm_at = al(at[0] + len(lst))
    perm = words[perm_at:perm_at + R]
    assert np.array_equal(np.sort(perm), np.arange(R))
    items = (R + 255) // 256
    off = perm_at + R
    for k in ks:
        ucap = al(S * min(256 * k, P))
        tn_at = al(off)
        tu_at = al(tn_at + items)
        tm_at = al(tu_at + items * ucap)
        off = tm_at + items * (ucap // 64) * 256 * 2
        masks = words[tm_at:off].view(np.uint64).reshape(items, ucap // 64, 256)
        for m in range(items):
            rows = perm[m * 256:(m + 1) * 256]
            keep = [set().union(*[set((f * V + ns + lists[u, f, :k]).tolist()) for f in range(S)]) for u in rows]
            union = np.array(sorted(set().union(*keep)), dtype=np.int64)
            U = int(words[tn_at + m])
            assert U == len(union), (k, m)
            assert np.array_equal(words[tu_at + m * ucap:tu_at + m * ucap + U], union), (k, m)
            bits = (masks[m][np.arange(U) // 64] >> (np.arange(U) % 64).astype(np.uint64)[:, None]) & np.uint64(1)
            want = np.zeros((U, 256), bool)
            pos = {t: e for e, t in enumerate(union.tolist())}
            for r, ks_r in enumerate(keep):
                want[[pos[t] for t in ks_r], r] = True
            assert np.array_equal(bits.astype(bool), want), (k, m)


def _check_token_heads(case, heads, att, sels, rows):
    """Per-frame lists of every token-wise head (the given query rows) against the oracle; each
    head is added to `sels`.  Returns {head: lists identical}."""
    hw = _hw()
    L = case.L
    exact = {}
    for h, hc in enumerate(heads):
        if hc.kind != TOKEN:
            continue
        lists = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).reshape(L.S * L.P, L.S, hc.k)
        exact[h] = check_token_lists(lists, L, sels.base.unit, hc.k, rows(h), f"token head {h}")
        sels.accept(L, h, hc, lists, exact[h])
    return exact


@pytest.mark.parametrize("name", list(TOKEN_CASES))
def test_token_heads_all_rows(name):
    hw = _hw()
    case = Case(TOKEN_CASES[name])
    heads = case.wl.heads
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    sels = check_selection(case, heads, att, sel)
    _check_token_heads(case, heads, att, sels, lambda h: np.arange(case.L.N))
    check_rows(case, heads, sels, out, lambda h: np.arange(case.L.N))
    pairs = hw.saf3r_kept_pairs(att.layout, att.cfg, att.cache)
    for h, hc in enumerate(heads):
        if hc.kind == TOKEN:
            assert int(pairs[h]) == sum(O.kept_count(case.L, hc, sels[h], h, i) for i in range(case.L.N))


@pytest.mark.parametrize("n_feat", [2, 5])
def test_token_heads_tied_features(n_feat):
    """Every patch takes one of n_feat DINO features, so a query's scores tie in large groups:
    with 2 features a frame's candidates overflow the short ranking (the general ranking runs),
    with 5 the short ranking sees whole tie groups; k = 40 always takes the general ranking.
    Ties go to the lower patch index on both sides, so the lists must be identical."""
    case = Case(_custom(3, 12, [HeadCfg(TOKEN, k=16), HeadCfg(TOKEN, k=5), HeadCfg(TOKEN, k=40),
                                HeadCfg(SCAN, stride=4, phase=1)]))
    L = case.L
    rng = np.random.default_rng(40 + n_feat)
    base = rng.standard_normal((n_feat, L.dino_dim)).astype(np.float32)
    case.dino = torch.from_numpy(np.ascontiguousarray(base[rng.integers(0, n_feat, size=L.S * L.P)])).cuda()
    heads = case.wl.heads
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    sels = check_selection(case, heads, att, sel)
    exact = _check_token_heads(case, heads, att, sels, lambda h: np.arange(L.N))
    assert all(exact[h] for h in range(3)), exact
    check_rows(case, heads, sels, out, lambda h: np.arange(L.N))


def test_token_heads_with_and_without_a_tensor_core_plan():
    """62 heads, 6 of them token-wise: the tensor-core kernel's plan array (64) holds the 62 heads'
    plans and the patch-query plans of only the first 2 token heads, so those 2 run their patch
    queries on the tensor cores over the cached unions while the other 4 run them in the gather
    kernel.  Every row of every head against the oracle."""
    heads = [HeadCfg(SCAN, stride=4, phase=h % 4) for h in range(56)] + \
            [HeadCfg(TOKEN, k=4), HeadCfg(TOKEN, k=9)] * 3
    case = Case(_custom(4, 10, heads, seed=95))
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    sels = check_selection(case, heads, att, sel)
    _check_token_heads(case, heads, att, sels, lambda h: np.arange(case.L.N))
    check_rows(case, heads, sels, out, lambda h: np.arange(case.L.N))


def test_s32_token_heads_sampled_rows(s32):
    """Per-frame Top-16 token-wise heads on the S=32 layer (the other heads as configured)."""
    heads = [HeadCfg(TOKEN, k=16)] * 4 + list(s32.wl.heads[4:])
    att, out = run_gpu(s32, heads, out_fp32=False)
    sel = oracle_select(s32, heads)
    sels = check_selection(s32, heads, att, sel)
    rows = {h: sample_rows(s32.wl, h, 64) for h in range(4)}
    _check_token_heads(s32, heads, att, sels, lambda h: rows[h])
    check_rows(s32, heads, sels, out, lambda h: rows[h] if h < 4 else sample_rows(s32.wl, h, 128))


# ---------------------------------------------------------------- running-max growth

def test_growing_logits_rescale_the_accumulator():
    """Every query gets q_0 = 8 and key j gets k_0 = 7 * floor(3j / N), so the logits of the middle
    and last third of the token sequence are raised by 7 and 14 (natural units, about 10 and 20
    in log2 units, each past the kernel's stale-max threshold of 8): every row's running max jumps
    twice, inside blocks as well as between them, and the accumulator and the partly written P
    are rescaled.  The softmax stays spread over a third of the keys (bf16 P rounding averages
    out).  All rows of every head kind against the oracle."""
    heads = [HeadCfg(PROBE, k=300), HeadCfg(SCAN, stride=2, phase=1), HeadCfg(DENSE), HeadCfg(POSITION),
             HeadCfg(CORR, k=6)]
    case = Case(_custom(4, 16, heads, seed=91))
    L = case.L
    step = torch.div(torch.arange(L.N, device="cuda") * 3, L.N, rounding_mode="floor").to(torch.float32)
    case.q[:, :, 0] = 8.0
    case.k[:, :, 0] = (7.0 * step).to(torch.bfloat16).view(1, L.N)
    case.Q, case.K = bf16_to_f32(case.q), bf16_to_f32(case.k)
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    sels = check_selection(case, heads, att, sel)
    check_rows(case, heads, sels, out, lambda h: np.arange(L.N))
