"""Head-sharded execution on one GPU: the ranks of a G-way split run one after another
(no collective, nothing waits on another launch).  Each rank's block is checked against the
oracle - its heads' exported index sets against the oracle's selection, its output rows
against the oracle's attention over those sets - and the blocks, put side by side, must
equal the unsharded layer bit for bit (every head's plan, items and arithmetic are the same
whichever heads share its launch)."""
import numpy as np
import pytest

import oracle as O
from saf3r_synth import WORKLOADS, Scene, bf16_to_f32, qkv, sample_rows
from parity_util import HeadSelections, check_probe, check_tiles, compare_outputs

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,world,rows", [("tiny", 2, 0), ("tiny", 4, 0), ("s32", 4, 128)])
def test_sharded_heads_match_the_oracle_and_the_full_layer(name, world, rows):
    import head_wise_dynamic_b200 as hw
    from head_wise_dynamic_b200.sharding import ShardedGlobalAttention
    wl = WORKLOADS[name]
    L = wl.layout
    scene = Scene(wl)
    q, k, v = qkv(scene, 0, device="cuda")
    dino = torch.from_numpy(scene.dino()).cuda()
    Q, K, V = (bf16_to_f32(t) for t in (q, k, v))
    sels = HeadSelections(O.select(L, wl.heads, Q, K, scene.dino()))
    full = hw.SparseGlobalAttention(L, wl.heads, out_dtype=torch.float32)
    full.select(q, k, dino)
    ref = full(q, k, v).clone()
    blocks = []
    for rank in range(world):
        sh = ShardedGlobalAttention(L, wl.heads, world=world, rank=rank, out_dtype=torch.float32)
        sh.select(q, k, dino)
        block = sh(q, k, v, gather=False).clone()
        torch.cuda.synchronize()
        hw.saf3r_check()
        blocks.append(block)
        o = block.cpu().numpy()
        for hl, h in enumerate(range(sh.h0, sh.h1)):
            hc = wl.heads[h]
            if hc.kind == O.PROBE:
                keys = hw.saf3r_cache_export(sh.att.layout, sh.att.cfg, sh.att.cache, hl)
                sels.accept(L, h, hc, keys, check_probe(keys, L, sels.base, h, hc.k, f"rank {rank} head {h}"))
            elif hc.kind in (O.CORR, O.HYBRID):
                ranked = hw.saf3r_cache_export(sh.att.layout, sh.att.cfg, sh.att.cache, hl).reshape(L.T, hc.k)
                sels.accept(L, h, hc, ranked, check_tiles(ranked, sels.base, hc.k, f"rank {rank} head {h}"))
            r = sample_rows(wl, h, rows) if rows else np.arange(L.N)
            want = O.sparse_rows(L, hc, sels[h], h, Q[h], K[h], V[h], r)
            compare_outputs(o[hl][r], want, f"rank {rank} of {world}, head {h}")
    sels.report(f"{name} split {world} ways")
    assert torch.equal(torch.cat(blocks, dim=0), ref)
