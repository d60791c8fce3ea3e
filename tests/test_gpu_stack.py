"""Profiling of the 24-layer stack's layout (S=64 views, N=87,936, H=16) on the GPU against
the oracle on sampled rows.

The stack picks, per head and per layer, the cheapest of ten candidate configurations whose
output NMSE against dense attention is at most 1e-2 (SAF3R, section 4.2).  At this size the
oracle cannot evaluate every row, so each NMSE the GPU measured over all rows is compared
with the oracle's ratio estimate on seeded row samples, within a bound derived from that
sample's own spread (the delta-method standard error of a ratio estimator: 5 standard
errors plus a small absolute floor); the kept-pair counts (Omega / 4d) are compared exactly,
and the choice wherever the sampled table decides it with a clear margin.
"""
import numpy as np
import pytest

import oracle as O
from saf3r_synth import SCAN, WORKLOADS, Scene, bf16_to_f32, qkv, sample_rows

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

NMSE_MAX = 1e-2
ROWS = 192         # sampled query rows per head for the oracle
Z = 5.0            # standard errors of the ratio estimate
ABS_FLOOR = 2e-5
MARGIN = 2.0       # a candidate is "clearly" in (out) when its estimate is below (above) NMSE_MAX / MARGIN (* MARGIN)


def _same(cfg, cand, h):
    phase = (h % cand.stride) if cand.kind == SCAN else cand.phase
    return (cfg.type, cfg.k, cfg.stride, cfg.phase) == (cand.kind, cand.k, cand.stride, phase)


def _ratio_and_se(err_rows, full_rows):
    """Ratio estimate sum(e)/sum(f) over the sampled rows and its delta-method standard error."""
    e = np.asarray(err_rows, dtype=np.float64)
    f = np.asarray(full_rows, dtype=np.float64)
    n = len(e)
    r = e.sum() / f.sum()
    resid = e - r * f
    se = np.sqrt((resid ** 2).sum() / (n - 1) / n) / f.mean()
    return r, se


@pytest.mark.parametrize("layer", [0, 12, 23])
def test_stack_layer_profile_matches_sampled_oracle(layer):
    import head_wise_dynamic_b200 as hw
    wl = WORKLOADS["stack"]
    L = wl.layout
    cands = wl.candidates
    scene = Scene(wl)
    q, k, v = qkv(scene, layer, device="cuda")
    dino_np = scene.dino()
    dino = torch.from_numpy(dino_np).cuda()
    Lc = hw.layout_of(L)
    ws = torch.empty(hw.saf3r_profile_workspace_bytes(Lc, cands), dtype=torch.uint8, device="cuda")
    chosen, nmse, pairs = hw.saf3r_profile_heads(Lc, cands, q, k, v, dino, NMSE_MAX, ws)
    torch.cuda.synchronize()
    hw.saf3r_check()
    assert np.all(np.isfinite(nmse)) and np.all(nmse >= 0.0)

    Q, K, V = (bf16_to_f32(t) for t in (q, k, v))
    rows = [sample_rows(wl, h, ROWS, seed_extra=100 + layer) for h in range(L.H)]
    full = [O.dense_rows(Q[h], K[h], V[h], rows[h]) for h in range(L.H)]
    ref = np.zeros((L.H, len(cands)))
    omega = np.zeros((L.H, len(cands)))
    worst = 0.0
    for c, cand in enumerate(cands):
        heads = [O.apply_candidate(cand, h) for h in range(L.H)]
        sel = O.select(L, heads, Q, K, dino_np)
        for h in range(L.H):
            p = O.kept_pairs(L, heads[h], sel, h)
            assert pairs[h, c] == p, (h, c, pairs[h, c], p)
            omega[h, c] = O.omega(L, p)
            sp = O.sparse_rows(L, heads[h], sel, h, Q[h], K[h], V[h], rows[h])
            r, se = _ratio_and_se(((full[h] - sp) ** 2).sum(axis=1), (full[h] ** 2).sum(axis=1))
            ref[h, c] = r
            dev = abs(nmse[h, c] - r)
            worst = max(worst, dev / (se + 1e-300))
            assert dev <= Z * se + ABS_FLOOR, (h, c, nmse[h, c], r, se)
    print(f"layer {layer}: largest |gpu - sample estimate| = {worst:.2f} standard errors")

    for h in range(L.H):
        got = [c for c in range(len(cands)) if _same(chosen[h], cands[c], h)]
        assert got, f"head {h}: chosen config is not a candidate"
        g = got[0]
        # the host rule applied to the GPU's own table and the exact Omega
        assert g == O.choose_config(nmse[h], omega[h], NMSE_MAX), (h, g, nmse[h], omega[h])
        # the choice is admissible by the full-row NMSE the GPU measured ...
        assert nmse[h, g] <= NMSE_MAX or np.all(nmse[h] > NMSE_MAX)
        # ... and no cheaper candidate is clearly admissible by the sampled oracle
        for c in range(len(cands)):
            if omega[h, c] < omega[h, g]:
                assert not ref[h, c] < NMSE_MAX / MARGIN, (h, c, g, ref[h], nmse[h])
        # a choice the sampled oracle clearly rules out is wrong
        if np.any(nmse[h] <= NMSE_MAX):
            assert not ref[h, g] > NMSE_MAX * MARGIN, (h, g, ref[h], nmse[h])
