"""Parity at the benchmark's full sizes, in the launch configuration bench.py times:
all index sets against the oracle, plus seeded sampled query rows per head (the
oracle computes them one group of equal key sets at a time)."""
import numpy as np
import pytest

import oracle as O
from saf3r_synth import WORKLOADS, Scene, bf16_to_f32, qkv, sample_rows
from parity_util import HeadSelections, check_probe, check_tiles, check_token_lists, compare_outputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _check_layer(wl, att, scene, layer, rows_per_head, sels=None):
    """One layer call: on the first call (sels None) every index set against the oracle, then the
    sampled rows of every head against the oracle over that head's validated set."""
    import head_wise_dynamic_b200 as hw
    L = wl.layout
    q, k, v = qkv(scene, layer, device="cuda")
    Q, K, V = (bf16_to_f32(t) for t in (q, k, v))
    if sels is None:
        att.select(q, k, torch.from_numpy(scene.dino()).cuda())
        sels = HeadSelections(O.select(L, wl.heads, Q, K, scene.dino()))
        for h, hc in enumerate(wl.heads):
            if hc.kind == O.PROBE:
                keys = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h)
                sels.accept(L, h, hc, keys, check_probe(keys, L, sels.base, h, hc.k, f"probe head {h}"))
            elif hc.kind in (O.CORR, O.HYBRID):  # ranked tiles
                ranked = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).reshape(L.T, hc.k)
                sels.accept(L, h, hc, ranked, check_tiles(ranked, sels.base, hc.k, f"tile head {h}"))
            elif hc.kind == O.TOKEN:  # per-frame lists of the rows that are checked below
                lists = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).reshape(L.S * L.P, L.S, hc.k)
                rows = sample_rows(wl, h, rows_per_head, seed_extra=layer)
                sels.accept(L, h, hc, lists, check_token_lists(lists, L, sels.base.unit, hc.k, rows,
                                                               f"token head {h}"))
    att.out.fill_(float("nan"))
    out = att(q, k, v)
    torch.cuda.synchronize()
    hw.saf3r_check()
    o = out.float().cpu().numpy()
    for h, hc in enumerate(wl.heads):
        rows = sample_rows(wl, h, rows_per_head, seed_extra=layer)
        ref = O.sparse_rows(L, hc, sels[h], h, Q[h], K[h], V[h], rows)
        compare_outputs(o[h][rows], ref, f"layer {layer} head {h}")
    sels.report(f"{wl.name} layer {layer}")
    assert np.isfinite(o).all(), "a row was not written"
    return sels


def test_s100_layer_and_cache_reuse():
    import head_wise_dynamic_b200 as hw
    wl = WORKLOADS["s100"]
    scene = Scene(wl)
    att = hw.SparseGlobalAttention(wl.layout, wl.heads)  # bf16 output, as timed
    sels = _check_layer(wl, att, scene, 0, 2048)
    # a later layer call with fresh Q/K/V reuses the cached sets
    _check_layer(wl, att, scene, wl.calls - 1, 256, sels=sels)


def test_s200_layer():
    import head_wise_dynamic_b200 as hw
    wl = WORKLOADS["s200"]
    scene = Scene(wl)
    att = hw.SparseGlobalAttention(wl.layout, wl.heads)
    _check_layer(wl, att, scene, 0, 1024)


def test_s100_hybrid_layer():
    """The S=100 layer with tile Top-64 united with a stride-32 lattice on the correspondence heads."""
    import head_wise_dynamic_b200 as hw
    wl = WORKLOADS["s100_hybrid"]
    scene = Scene(wl)
    att = hw.SparseGlobalAttention(wl.layout, wl.heads)
    _check_layer(wl, att, scene, 0, 512)


def test_s100_token_layer():
    """The S=100 layer with per-frame Top-16 token-wise heads in place of the position heads:
    sampled rows (the special-token rows among them run in the tensor-core kernel as dense rows,
    the patch rows in the gather kernel) and their per-frame lists against the oracle."""
    import head_wise_dynamic_b200 as hw
    wl = WORKLOADS["s100_token"]
    scene = Scene(wl)
    att = hw.SparseGlobalAttention(wl.layout, wl.heads)
    _check_layer(wl, att, scene, 0, 96)
