"""The allocation-free index build, saf3r_select_kv_static, against saf3r_select_kv.

Callers that cannot allocate device memory (allocator-free latency loops, hosts
that pass only inputs and outputs) use the
static entry point; it must build the same cache as the regular one.  This file
is collected last so that a failure here comes after every other test ran."""
import numpy as np
import pytest

from parity_util import compare_outputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _workload(name):
    from saf3r_synth import CORR, PROBE, TOKEN, WORKLOADS, HeadCfg, Layout, Workload
    if name == "tiny_token":
        # token-wise heads (two per-frame budgets) beside a probe and a correspondence head
        return Workload("tiny_token", Layout(S=4, g=16, H=4), M=512, delta=37, D=256,
                        heads=[HeadCfg(TOKEN, k=8), HeadCfg(PROBE, k=128), HeadCfg(CORR, k=4), HeadCfg(TOKEN, k=4)],
                        seed=1234)
    return WORKLOADS[name]


def _inputs(name):
    from saf3r_synth import Scene, qkv
    wl = _workload(name)
    scene = Scene(wl)
    q, k, v = qkv(scene, 0, device="cuda")
    return wl, q, k, v, torch.from_numpy(scene.dino()).cuda()


@pytest.mark.parametrize("name", ["tiny", "s32", "tiny_token"])
def test_static_select_matches_regular_on_two_calls(name):
    import head_wise_dynamic_b200 as hw
    from saf3r_synth import CORR, PROBE, TOKEN
    wl, q, k, v, dino = _inputs(name)
    L = hw.layout_of(wl.layout)
    cfg = hw.cfg_array(wl.heads)
    cb = hw.saf3r_cache_bytes(L, cfg)
    ref = torch.empty(cb, dtype=torch.uint8, device="cuda")
    ws = torch.empty(max(hw.saf3r_workspace_bytes(L, cfg, hw.OP_SELECT),
                         hw.saf3r_workspace_bytes(L, cfg, hw.OP_SPARSE)), dtype=torch.uint8, device="cuda")
    hw.saf3r_select_kv(L, cfg, q, k, dino, ref, ws)
    out_ref = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    hw.saf3r_sparse_attn(L, cfg, ref, q, k, v, out_ref, ws)
    torch.cuda.synchronize()
    hw.saf3r_check()
    for call in range(2):
        cache = torch.full((cb,), 0xAB, dtype=torch.uint8, device="cuda")  # no help from a previous cache
        hw.saf3r_select_kv_static(L, cfg, q, k, dino, cache)
        torch.cuda.synchronize()
        hw.saf3r_check()
        for h, hc in enumerate(wl.heads):
            if hc.kind in (PROBE, CORR, TOKEN):
                a = hw.saf3r_cache_export(L, cfg, cache, h)
                b = hw.saf3r_cache_export(L, cfg, ref, h)
                assert np.array_equal(a, b), f"call {call}: head {h} index list differs"
        out = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
        hw.saf3r_sparse_attn(L, cfg, cache, q, k, v, out, ws)
        torch.cuda.synchronize()
        hw.saf3r_check()
        for h in range(L.H):
            compare_outputs(out[h].cpu().numpy(), out_ref[h].cpu().numpy(), f"call {call} head {h}")


def test_static_select_rejects_layers_beyond_its_scratch():
    import head_wise_dynamic_b200 as hw
    from saf3r_synth import CORR, PROBE, HeadCfg, Layout
    big = Layout(S=400, g=37, H=8)  # T = 8588 tiles: 51 MiB of select workspace
    heads = [HeadCfg(PROBE, k=1000)] * 4 + [HeadCfg(CORR, k=64)] * 4
    L = hw.layout_of(big)
    cfg = hw.cfg_array(heads)
    assert hw.saf3r_workspace_bytes(L, cfg, hw.OP_SELECT) > 40 << 20
    dummy = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(hw.Saf3rError) as e:
        hw.saf3r_select_kv_static(L, cfg, dummy, dummy, dummy, dummy)
    assert e.value.status == hw.ERR_UNSUPPORTED
