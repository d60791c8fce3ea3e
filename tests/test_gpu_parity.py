"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Index sets must match exactly up to the boundary band;
outputs within max-abs 1e-2 and rel-L2 5e-3."""
import numpy as np
import pytest

import oracle as O
from saf3r_synth import (CORR, DENSE, HYBRID, POSITION, PROBE, SCAN, TOKEN, WORKLOADS, HeadCfg, Layout, Scene,
                         Workload, bf16_to_f32, qkv, sample_rows)
from parity_util import check_probe, check_tiles, check_token_lists, compare_outputs

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
    hw = _hw()
    exact = {}
    for h, hc in enumerate(heads):
        if hc.kind == PROBE:
            keys = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h)
            exact[h] = check_probe(keys, case.L, sel, h, hc.k, f"probe head {h}")
        elif hc.kind in (CORR, HYBRID):
            ranked = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).reshape(case.L.T, hc.k)
            exact[h] = check_tiles(ranked, sel, hc.k, f"tile head {h}")
    return exact


def check_rows(case, heads, sel, out, rows_per_head, exact):
    out = out.float().cpu().numpy()
    for h, hc in enumerate(heads):
        if not exact.get(h, True):
            continue  # a boundary tie was resolved differently: the set is valid but not unique
        rows = rows_per_head(h)
        ref = O.sparse_rows(case.L, hc, sel, h, case.Q[h], case.K[h], case.V[h], rows)
        compare_outputs(out[h][rows], ref, f"head {h} ({hc.kind})")


@pytest.fixture(scope="module")
def tiny():
    return Case(WORKLOADS["tiny"])


@pytest.mark.parametrize("out_fp32", [True, False])
def test_tiny_all_rows(tiny, out_fp32):
    heads = tiny.wl.heads
    att, out = run_gpu(tiny, heads, out_fp32)
    sel = oracle_select(tiny, heads)
    exact = check_selection(tiny, heads, att, sel)
    check_rows(tiny, heads, sel, out, lambda h: np.arange(tiny.L.N), exact)


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


def _custom(S, g, heads, seed=7, M=256, D=128):
    L = Layout(S=S, g=g, H=len(heads))
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
    exact = check_selection(case, heads, att, sel)
    check_rows(case, heads, sel, out, lambda h: np.arange(case.L.N), exact)


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
    exact = check_selection(s32, heads, att, sel)
    check_rows(s32, heads, sel, out, lambda h: sample_rows(s32.wl, h, 512), exact)


def test_s32_hybrid_heads_sampled_rows_and_pairs(s32):
    """Tile Top-32 united with stride-20 lattices (phase = head mod 20) on the S=32 layer."""
    hw = _hw()
    heads = [HeadCfg(HYBRID, k=32, stride=20, phase=h % 20) for h in range(s32.L.H)]
    att, out = run_gpu(s32, heads, out_fp32=False)
    sel = oracle_select(s32, heads)
    exact = check_selection(s32, heads, att, sel)
    check_rows(s32, heads, sel, out, lambda h: sample_rows(s32.wl, h, 256), exact)
    pairs = hw.saf3r_kept_pairs(att.layout, att.cfg, att.cache)
    for h in (0, 7):
        if exact.get(h, True):
            assert int(pairs[h]) == O.kept_pairs(s32.L, heads[h], sel, h)


# ---------------------------------------------------------------- token-wise per-frame DINO Top-K

TOKEN_CASES = {
    # ragged layout; k = P keeps every key; k = 1; a main-kernel head beside them
    "token_ragged": _custom(3, 9, [HeadCfg(TOKEN, k=3), HeadCfg(TOKEN, k=81), HeadCfg(TOKEN, k=1),
                                   HeadCfg(SCAN, stride=5, phase=4)]),
    # token-wise heads mixed with the other kinds in one call
    "token_mixed": _custom(4, 16, [HeadCfg(TOKEN, k=16), HeadCfg(CORR, k=4), HeadCfg(TOKEN, k=5),
                                   HeadCfg(POSITION)], D=256),
}


def _check_token_heads(case, heads, att, sel, rows):
    hw = _hw()
    L = case.L
    exact = {}
    for h, hc in enumerate(heads):
        if hc.kind != TOKEN:
            continue
        lists = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).reshape(L.S * L.P, L.S, hc.k)
        exact[h] = check_token_lists(lists, L, sel.unit, hc.k, rows, f"token head {h}")
    return exact


@pytest.mark.parametrize("name", list(TOKEN_CASES))
def test_token_heads_all_rows(name):
    hw = _hw()
    case = Case(TOKEN_CASES[name])
    heads = case.wl.heads
    att, out = run_gpu(case, heads)
    sel = oracle_select(case, heads)
    exact = check_selection(case, heads, att, sel)
    exact.update(_check_token_heads(case, heads, att, sel, np.arange(case.L.N)))
    check_rows(case, heads, sel, out, lambda h: np.arange(case.L.N), exact)
    pairs = hw.saf3r_kept_pairs(att.layout, att.cfg, att.cache)
    for h, hc in enumerate(heads):
        if hc.kind == TOKEN:
            assert int(pairs[h]) == sum(O.kept_count(case.L, hc, sel, h, i) for i in range(case.L.N))


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
    exact = check_selection(case, heads, att, sel)
    exact.update(_check_token_heads(case, heads, att, sel, np.arange(L.N)))
    assert all(exact[h] for h in range(3)), exact
    check_rows(case, heads, sel, out, lambda h: np.arange(L.N), exact)


def test_s32_token_heads_sampled_rows(s32):
    """Per-frame Top-16 token-wise heads on the S=32 layer (the other heads as configured)."""
    heads = [HeadCfg(TOKEN, k=16)] * 4 + list(s32.wl.heads[4:])
    att, out = run_gpu(s32, heads, out_fp32=False)
    sel = oracle_select(s32, heads)
    exact = check_selection(s32, heads, att, sel)
    rows = {h: sample_rows(s32.wl, h, 64) for h in range(4)}
    hw = _hw()
    L = s32.L
    for h in range(4):
        lists = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).reshape(L.S * L.P, L.S, 16)
        exact[h] = check_token_lists(lists, L, sel.unit, 16, rows[h], f"token head {h}")
    check_rows(s32, heads, sel, out, lambda h: rows[h] if h < 4 else sample_rows(s32.wl, h, 128), exact)
