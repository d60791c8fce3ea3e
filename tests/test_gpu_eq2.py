"""GPU parity of the eq. 2 search (section 4.2: progressive substitution from a
uniform-stride baseline, error averaged over a calibration set) against the
oracle, on a layout small enough for the oracle to use every row."""
import numpy as np
import pytest

import oracle as O
from saf3r_synth import CORR, HYBRID, POSITION, PROBE, SCAN, HeadCfg, Layout, Scene, Workload, bf16_to_f32, qkv

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SIGMA = 0.85


def test_eq2_search_matches_oracle():
    import head_wise_dynamic_b200 as hw
    L = Layout(S=4, g=16, H=4)
    wl = Workload("eq2", L, M=256, delta=37, D=128, heads=[HeadCfg(POSITION)] * 4, seed=5151)
    base_stride = hw.baseline_stride(SIGMA)
    assert base_stride == O.baseline_stride(SIGMA) == 7
    cands = [HeadCfg(SCAN, stride=base_stride), HeadCfg(POSITION), HeadCfg(PROBE, k=64), HeadCfg(PROBE, k=128),
             HeadCfg(CORR, k=1), HeadCfg(CORR, k=2), HeadCfg(SCAN, stride=8), HeadCfg(SCAN, stride=16),
             HeadCfg(HYBRID, k=1, stride=16)]
    scene = Scene(wl)
    dino_np = scene.dino()
    dino = torch.from_numpy(dino_np).cuda()
    inputs = [tuple(qkv(scene, layer, device="cuda")) + (dino,) for layer in range(2)]
    Lc = hw.layout_of(L)
    ws = torch.empty(hw.saf3r_profile_workspace_bytes(Lc, cands), dtype=torch.uint8, device="cuda")
    choice, mean, pairs = hw.profile_heads_eq2(Lc, cands, 0, inputs, ws)
    torch.cuda.synchronize()
    hw.saf3r_check()

    tables, costs = [], []
    for q, k, v, _ in inputs:
        Q, K, V = (bf16_to_f32(t) for t in (q, k, v))
        tables.append(O.nmse_table_sampled(L, cands, Q, K, V, dino_np, [np.arange(L.N)] * L.H))
        cost = np.zeros((L.H, len(cands)), dtype=np.int64)
        for c, cand in enumerate(cands):
            heads = [O.apply_candidate(cand, h) for h in range(L.H)]
            sel = O.select(L, heads, Q, K, dino_np)
            for h in range(L.H):
                cost[h, c] = O.kept_pairs(L, heads[h], sel, h)
        costs.append(cost)
    assert np.array_equal(pairs, np.stack(costs)), (pairs, np.stack(costs))
    ref_mean = np.mean(tables, axis=0)
    assert np.all(np.abs(mean - ref_mean) <= 1e-2 * ref_mean + 2e-5), (mean, ref_mean)
    want = O.choose_eq2(tables, costs, 0)
    for h in range(L.H):
        if choice[h] != want[h]:
            # a choice decided by errors within 1% of each other may go either way
            a, b = ref_mean[h, choice[h]], ref_mean[h, want[h]]
            assert abs(a - b) <= 1e-2 * max(a, b), (h, choice[h], want[h], ref_mean[h])
    # the choice never costs more than the baseline, nor errs more (on the GPU's own table)
    W = np.stack(costs).mean(axis=0)
    for h in range(L.H):
        assert W[h, choice[h]] <= W[h, 0] and mean[h, choice[h]] <= mean[h, 0]
