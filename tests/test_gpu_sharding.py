"""Head-sharded execution on one GPU: the ranks of a G-way split run one after another
(no collective, nothing waits on another launch) and their local blocks, put side by
side, must equal the unsharded layer bit for bit - every head's plan, items and
arithmetic are the same whichever heads share its launch."""
import pytest

from saf3r_synth import WORKLOADS, Scene, qkv

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,world", [("tiny", 2), ("tiny", 4), ("s32", 4)])
def test_sharded_heads_equal_the_full_layer(name, world):
    import head_wise_dynamic_b200 as hw
    from head_wise_dynamic_b200.sharding import ShardedGlobalAttention
    wl = WORKLOADS[name]
    scene = Scene(wl)
    q, k, v = qkv(scene, 0, device="cuda")
    dino = torch.from_numpy(scene.dino()).cuda()
    full = hw.SparseGlobalAttention(wl.layout, wl.heads, out_dtype=torch.float32)
    full.select(q, k, dino)
    ref = full(q, k, v).clone()
    blocks = []
    for rank in range(world):
        sh = ShardedGlobalAttention(wl.layout, wl.heads, world=world, rank=rank, out_dtype=torch.float32)
        sh.select(q, k, dino)
        blocks.append(sh(q, k, v, gather=False).clone())
    torch.cuda.synchronize()
    hw.saf3r_check()
    assert torch.equal(torch.cat(blocks, dim=0), ref)
