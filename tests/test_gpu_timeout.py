"""The timeout path of the bounded device waits, on the GPU without a fault: one softmax
warp withholds one arrival (a test hook of the library), so the tensor-core warp's wait for
it runs out after a short budget.  The kernel must report SAF3R_ERR_TIMEOUT through
saf3r_check, leave the context usable, and the very next call must run normally."""
import numpy as np
import pytest

import oracle as O
from saf3r_synth import WORKLOADS, Scene, bf16_to_f32, qkv
from parity_util import HeadSelections, check_probe, check_tiles, compare_outputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

SHORT_BUDGET = 20_000_000  # clock cycles (~10 ms at 1.965 GHz)


@pytest.mark.parametrize("dense", [False, True])
def test_expired_wait_is_reported_and_the_next_call_is_clean(dense):
    import head_wise_dynamic_b200 as hw
    wl = WORKLOADS["tiny"]
    L = wl.layout
    scene = Scene(wl)
    q, k, v = qkv(scene, 0, device="cuda")
    dino = torch.from_numpy(scene.dino()).cuda()
    att = hw.SparseGlobalAttention(L, wl.heads, out_dtype=torch.float32)
    att.select(q, k, dino)
    wsd = torch.empty(hw.saf3r_workspace_bytes(att.layout, None, hw.OP_DENSE), dtype=torch.uint8, device="cuda")
    out = torch.empty((L.H, L.N, 64), dtype=torch.float32, device="cuda")

    def run():
        if dense:
            hw.saf3r_dense_attn(att.layout, q, k, v, out, wsd)
        else:
            att(q, k, v, out=out)

    torch.cuda.synchronize()
    hw.saf3r_check()
    hw.saf3r_set_wait_budget(SHORT_BUDGET)
    try:
        hw.saf3r_test_withhold_arrive()
        run()
        with pytest.raises(hw.Saf3rError) as e:
            hw.saf3r_check()
        assert e.value.status == hw.ERR_TIMEOUT
        hw.saf3r_check()  # the error word was cleared
        # the same short budget, no withheld arrival: a normal call finishes well inside it
        out.fill_(float("nan"))
        run()
        hw.saf3r_check()
    finally:
        hw.saf3r_set_wait_budget(0)
    o = out.cpu().numpy()
    Q, K, V = (bf16_to_f32(t) for t in (q, k, v))
    rows = np.arange(L.N)
    if dense:
        for h in range(L.H):
            compare_outputs(o[h], O.dense_rows(Q[h], K[h], V[h], rows), f"dense head {h} after a timeout")
        return
    sels = HeadSelections(O.select(L, wl.heads, Q, K, scene.dino()))
    for h, hc in enumerate(wl.heads):
        if hc.kind == O.PROBE:
            keys = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h)
            sels.accept(L, h, hc, keys, check_probe(keys, L, sels.base, h, hc.k, f"probe head {h}"))
        elif hc.kind in (O.CORR, O.HYBRID):
            ranked = hw.saf3r_cache_export(att.layout, att.cfg, att.cache, h).reshape(L.T, hc.k)
            sels.accept(L, h, hc, ranked, check_tiles(ranked, sels.base, hc.k, f"tile head {h}"))
        ref = O.sparse_rows(L, hc, sels[h], h, Q[h], K[h], V[h], rows)
        compare_outputs(o[h], ref, f"head {h} after a timeout")
