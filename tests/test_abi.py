"""The C-ABI library loads, exports every symbol include/saf3r.h declares, and
rejects bad arguments on the host (no GPU needed: no compute call is made)."""
import ctypes

import numpy as np
import pytest

import head_wise_dynamic_b200 as hw
from saf3r_synth import CORR, PROBE, SCAN, TOKEN, WORKLOADS, HeadCfg


def test_library_exports_every_declared_symbol():
    names = hw.header_functions()
    assert "saf3r_select_kv" in names and "saf3r_sparse_attn" in names
    L = hw.lib()
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings():
    for s in range(6):
        assert hw.status_string(s)


def _tiny():
    wl = WORKLOADS["tiny"]
    return hw.layout_of(wl.layout), hw.cfg_array(wl.heads)


def test_sizes_on_host():
    L, cfg = _tiny()
    cb = hw.saf3r_cache_bytes(L, cfg)
    # header (512 B) + 128 probe keys + T*kmax corr tiles (T = 17, kmax = 4)
    assert cb >= 512 + 128 * 4 + 17 * 4 * 4
    assert hw.saf3r_workspace_bytes(L, cfg, hw.OP_SELECT) > 0
    assert hw.saf3r_workspace_bytes(L, cfg, hw.OP_SPARSE) > 0
    assert hw.saf3r_workspace_bytes(L, None, hw.OP_DENSE) > 0


@pytest.mark.parametrize("field,value", [("d", 128), ("tile", 32), ("H", 0), ("H", 65), ("S", 0),
                                         ("n_special", 64), ("dino_dim", 6)])
def test_bad_layout_sizes_zero(field, value):
    L, cfg = _tiny()
    setattr(L, field, value)
    assert hw.saf3r_cache_bytes(L, cfg) == 0


@pytest.mark.parametrize("h,field,value", [(1, "k", 0), (1, "k", 10 ** 6), (2, "k", 18), (3, "stride", 0),
                                           (3, "phase", 8), (0, "radius", 4), (0, "radius", -2), (0, "type", 9)])
def test_bad_cfg_sizes_zero(h, field, value):
    L, cfg = _tiny()
    setattr(cfg[h], field, value)
    assert hw.saf3r_cache_bytes(L, cfg) == 0


def test_calls_reject_bad_arguments_before_any_launch():
    L, cfg = _tiny()
    lib = hw.lib()
    # null device pointers
    assert lib.saf3r_select_kv(ctypes.byref(L), cfg, None, None, None, None, None, None) == hw.ERR_INVALID
    assert lib.saf3r_sparse_attn(ctypes.byref(L), cfg, None, None, None, None, None, 0, None, None) == hw.ERR_INVALID
    # misaligned pointers
    bad = 0x1008
    assert lib.saf3r_dense_attn(ctypes.byref(L), bad, bad, bad, bad, 0, bad, None) == hw.ERR_INVALID
    # head dimension other than 64 is unsupported
    L.d = 128
    assert lib.saf3r_dense_attn(ctypes.byref(L), 0x1000, 0x1000, 0x1000, 0x1000, 0, 0x1000, None) == \
        hw.ERR_UNSUPPORTED


def test_choose_eq2_host_rule_matches_oracle():
    """saf3r_choose_eq2 is host logic: the C rule against the oracle on random tables."""
    import oracle as O
    rng = np.random.default_rng(11)
    for _ in range(100):
        n_in, H, C = int(rng.integers(1, 4)), int(rng.integers(1, 6)), int(rng.integers(1, 9))
        E = rng.choice([0.01, 0.02, 0.05, 0.1], size=(n_in, H, C)) * rng.choice([1.0, 1.5], size=(n_in, H, C))
        W = rng.integers(1, 6, size=(n_in, H, C)).astype(np.int64) * 1000
        base = int(rng.integers(0, C))
        choice, mean = hw.saf3r_choose_eq2(E, W, base)
        assert choice.tolist() == O.choose_eq2(E, W, base)
        assert np.allclose(mean, E.mean(axis=0), rtol=0, atol=1e-15)


def test_choose_eq2_rejects_bad_arguments():
    E = np.zeros((1, 2, 3))
    W = np.zeros((1, 2, 3), dtype=np.int64)
    with pytest.raises(hw.Saf3rError):
        hw.saf3r_choose_eq2(E, W, 3)
    with pytest.raises(hw.Saf3rError):
        hw.saf3r_choose_eq2(E, W, -1)
    assert hw.baseline_stride(0.85) == 7


@pytest.mark.parametrize("field,value", [("k", 0), ("k", 18), ("stride", 0), ("phase", 8), ("phase", -1)])
def test_bad_hybrid_cfg_sizes_zero(field, value):
    L, cfg = _tiny()
    cfg[2].type = hw.HYBRID
    cfg[2].k, cfg[2].stride, cfg[2].phase = 3, 8, 5
    assert hw.saf3r_cache_bytes(L, cfg) > 0
    setattr(cfg[2], field, value)
    assert hw.saf3r_cache_bytes(L, cfg) == 0


def test_token_cfg_validation():
    L, cfg = _tiny()
    cfg[2].type = hw.TOKEN
    cfg[2].k = 16
    assert hw.saf3r_cache_bytes(L, cfg) > 0
    for k in (0, L.grid_h * L.grid_w + 1):
        cfg[2].k = k
        assert hw.saf3r_cache_bytes(L, cfg) == 0
    cfg[2].k = 4
    L.dino_dim = 388  # beyond what the token-wise selection keeps in registers: unsupported
    assert hw.saf3r_cache_bytes(L, cfg) == 0


@pytest.mark.parametrize("S", [4, 32, 100])
def test_token_select_workspace_on_host(S):
    """Token-wise heads add to the select workspace: fp32 and fp16 unit features of the R = S*P
    patch tokens and the fp16 scores of one chunk of query rows, at most 1 GiB of them (every
    chunk a multiple of 128 rows, or all R rows), and the query order's buckets (3P + 1 ints) and
    sort keys (R 64-bit words)."""
    from saf3r_synth import Layout
    L = hw.layout_of(Layout(S=S, g=37 if S > 4 else 16, H=4))
    base = [HeadCfg(PROBE, k=64), HeadCfg(CORR, k=4), HeadCfg(SCAN, stride=4, phase=1), HeadCfg(SCAN, stride=8)]
    tok = [HeadCfg(PROBE, k=64), HeadCfg(CORR, k=4), HeadCfg(TOKEN, k=16), HeadCfg(SCAN, stride=8)]
    w0 = hw.saf3r_workspace_bytes(L, hw.cfg_array(base), hw.OP_SELECT)
    w1 = hw.saf3r_workspace_bytes(L, hw.cfg_array(tok), hw.OP_SELECT)
    R = L.S * L.grid_h * L.grid_w
    ld = (R + 7) // 8 * 8
    feats = R * L.dino_dim * 4 + R * ((L.dino_dim + 63) // 64 * 64) * 2
    chunk = min(R, max(128, (1 << 30) // (2 * ld) // 128 * 128))
    P = L.grid_h * L.grid_w
    order = (3 * P + 1 + 63) // 64 * 64 * 4 + R * 8
    assert w1 - w0 >= feats + chunk * ld * 2 + order
    assert w1 - w0 <= feats + min(R * ld * 2, (1 << 30)) + order + 4096


def test_baseline_stride_rule_in_the_library():
    import oracle as O
    for sigma in (0.0, 0.5, 0.75, 0.8, 0.85, 0.875, 0.9, 0.95, 0.96875, 0.99):
        assert hw.saf3r_baseline_stride(sigma) == O.baseline_stride(sigma), sigma
    assert hw.saf3r_baseline_stride(0.85) == 7  # section 5.1's sigma
    for bad in (-0.1, 1.0, 1.5, float("nan")):
        assert hw.lib().saf3r_baseline_stride(bad) == -1


def test_static_select_returns_the_regular_entry_points_codes():
    """saf3r_select_kv_static validates like saf3r_select_kv (before any device work)."""
    L, cfg = _tiny()
    f = hw.lib().saf3r_select_kv_static
    f.argtypes = [ctypes.POINTER(hw.saf3r_layout), ctypes.POINTER(hw.saf3r_head_cfg)] + [ctypes.c_void_p] * 5
    f.restype = ctypes.c_int
    p = 0x1000
    L.d = 128
    assert f(ctypes.byref(L), cfg, p, p, p, p, None) == hw.ERR_UNSUPPORTED
    L, cfg = _tiny()
    cfg[1].k = 0
    assert f(ctypes.byref(L), cfg, p, p, p, p, None) == hw.ERR_INVALID
    L, cfg = _tiny()
    L.dino_dim = 512
    tok = hw.cfg_array([HeadCfg(TOKEN, k=4)] + list(WORKLOADS["tiny"].heads[1:]))
    assert f(ctypes.byref(L), tok, p, p, p, p, None) == hw.ERR_UNSUPPORTED


def test_profile_rejects_a_token_candidate_without_dino():
    L, _ = _tiny()
    cand = hw.cfg_array([HeadCfg(TOKEN, k=4), HeadCfg(SCAN, stride=4)])
    lib = hw.lib()
    H = L.H
    chosen = (hw.saf3r_head_cfg * H)()
    nmse = (ctypes.c_double * (H * 2))()
    pairs = (ctypes.c_int64 * (H * 2))()
    p = 0x1000
    assert lib.saf3r_profile_heads(ctypes.byref(L), cand, 2, p, p, p, None, 0.01, chosen, nmse, pairs, p,
                                   None) == hw.ERR_INVALID


@pytest.mark.parametrize("S,g,on", [(4, 16, True), (200, 37, False)])
def test_token_cache_bytes_follow_the_documented_placement(S, g, on):
    """The cache size of a layer with token-wise heads, added up from the documented placement:
    header, probe lists, ranked tile lists and their order, the per-frame lists, then (when the
    unions fit: at most 2^28 union entries per budget) the patch query order and, per distinct k,
    union lengths, unions and masks, each region on a 64-word boundary.  S=200 at 37x37 patches
    and k=16 needs 2.9e8 union entries: no unions (the gather kernel takes those heads)."""
    from saf3r_synth import Layout
    heads = [HeadCfg(TOKEN, k=16), HeadCfg(CORR, k=4), HeadCfg(TOKEN, k=5), HeadCfg(PROBE, k=100)]
    lay = Layout(S=S, g=g, H=4)
    L = hw.layout_of(lay)
    al = lambda x: (x + 63) // 64 * 64
    ints = 512 // 4 + al(100)                      # header, the probe head's list
    ints += lay.T * 4 + lay.T                      # ranked tiles (kmax 4), their grouping order
    ints = al(ints) + lay.S * lay.P * lay.S * 16   # per-frame lists, tok_kmax 16
    R = lay.S * lay.P
    items = (R + 255) // 256
    if on:
        ints = al(ints) + R
        for k in (16, 5):
            ucap = al(lay.S * min(256 * k, lay.P))
            ints = al(ints) + items
            ints = al(ints) + items * ucap
            ints = al(ints) + items * (ucap // 64) * 256 * 2
    else:
        assert items * al(lay.S * min(256 * 5, lay.P)) > (1 << 28)
    assert hw.saf3r_cache_bytes(L, hw.cfg_array(heads)) == (ints * 4 + 255) // 256 * 256
