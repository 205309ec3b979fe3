"""Host-side logic of layer.py on the CPU: the tensor-parallel shard's weight slices."""
import pytest
import torch

from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import inputs as I
from fp8_block_scaled_biased_b200.layer import MoELayer


def _random_layer(cfg):
    layer = MoELayer(cfg, "cpu", tiled=False)
    g = torch.Generator().manual_seed(3)
    for t in (layer.w1, layer.w2):
        t.view(torch.uint8).copy_(torch.randint(0, 256, t.shape, generator=g, dtype=torch.uint8))
    for t in (layer.w1_scale, layer.w2_scale):
        t.copy_(torch.rand(t.shape, generator=g))
    return layer


@pytest.mark.parametrize("n", [2, 4])
def test_tp_shard_takes_the_gate_up_rows_and_down_columns_of_its_slice(n):
    cfg = I.MoEConfig("host_tp", T=4, H=256, E=3, G=1, TG=1, K=2, I=512)
    layer = _random_layer(cfg)
    Is = cfg.I // n
    for r in range(n):
        sh = layer.tp_shard(r, n)
        assert sh.cfg.I == Is and sh.w1.shape == (cfg.E, 2 * Is, cfg.H) and sh.w2.shape == (cfg.E, cfg.H, Is)
        for e in range(cfg.E):
            for i in range(Is):                       # row by row: gate row r*Is+i, up row I+r*Is+i
                assert torch.equal(sh.w1[e, i].view(torch.uint8), layer.w1[e, r * Is + i].view(torch.uint8))
                assert torch.equal(sh.w1[e, Is + i].view(torch.uint8), layer.w1[e, cfg.I + r * Is + i].view(torch.uint8))
            assert torch.equal(sh.w2[e].view(torch.uint8), layer.w2[e, :, r * Is:(r + 1) * Is].view(torch.uint8))
            for j in range(Is // 128):
                assert torch.equal(sh.w1_scale[e, j], layer.w1_scale[e, (r * Is) // 128 + j])
                assert torch.equal(sh.w1_scale[e, Is // 128 + j], layer.w1_scale[e, (cfg.I + r * Is) // 128 + j])
                assert torch.equal(sh.w2_scale[e, :, j], layer.w2_scale[e, :, (r * Is) // 128 + j])


def _tile(w):
    """The tiled layout by its definition (block (e, nb, kb) = rows nb*128.., columns kb*128..,
    row-major inside the block), written with a reshape and a permutation."""
    E, N, K = w.shape
    return w.view(torch.uint8).view(E, N // 128, 128, K // 128, 128).permute(0, 1, 3, 2, 4).contiguous()


@pytest.mark.parametrize("n", [2, 4])
def test_tiled_tp_shard_equals_the_tiled_row_major_shard(n):
    cfg = I.MoEConfig("host_tp", T=4, H=256, E=3, G=1, TG=1, K=2, I=512)
    rm = _random_layer(cfg)
    tl = MoELayer(cfg, "cpu", tiled=True)
    assert tl.w1.shape == (cfg.E, 2 * cfg.I // 128, cfg.H // 128, 128, 128)
    tl.w1.view(torch.uint8).copy_(_tile(rm.w1))
    tl.w2.view(torch.uint8).copy_(_tile(rm.w2))
    tl.w1_scale.copy_(rm.w1_scale)
    tl.w2_scale.copy_(rm.w2_scale)
    for r in range(n):
        a, b = rm.tp_shard(r, n), tl.tp_shard(r, n)
        assert b.tiled and b.cfg == a.cfg
        assert torch.equal(b.w1.view(torch.uint8), _tile(a.w1))
        assert torch.equal(b.w2.view(torch.uint8), _tile(a.w2))
        assert torch.equal(b.w1_scale, a.w1_scale) and torch.equal(b.w2_scale, a.w2_scale)


def test_tp_shard_rejects_a_split_inside_a_128_block():
    layer = MoELayer(I.TINY, "cpu")                    # I = 128: one block
    with pytest.raises(ValueError):
        layer.tp_shard(0, 2)
    with pytest.raises(ValueError):
        layer.tp_shard(1, 1)


def test_launches_per_forward_counts_the_sort_kernels():
    assert MoELayer(I.TINY, "cpu").launches_per_forward == 8            # 64 pairs: one sort kernel
    big = I.MoEConfig("host_big", T=200, H=256, E=16, G=4, TG=2, K=8, I=128)
    assert MoELayer(big, "cpu").launches_per_forward == 9               # 1600 pairs: count + scatter
