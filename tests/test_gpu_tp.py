"""GPU parity of the tensor-parallel shards of the layer (the pages' TP8 deployment, split
over the intermediate dimension I) against the CPU oracle: each rank's partial output, and
the ranks' sum against the whole layer."""
import pytest
import torch

from oracle import fp8moe_oracle as O
from fp8_block_scaled_biased_b200 import binding as B
from fp8_block_scaled_biased_b200 import inputs as I
from fp8_block_scaled_biased_b200.layer import MoELayer
from tests.gpu_helpers import assert_moe_close, full_size_tokens, oracle_expert, oracle_moe_rows

pytestmark = pytest.mark.gpu
DEV = "cuda"
MID = I.MoEConfig("mid_t256_h1024_e32", T=256, H=1024, E=32, G=4, TG=2, K=4, I=512, seed=1)
ODD = I.MoEConfig("odd_t37_h640_e24_k5", T=37, H=640, E=24, G=4, TG=3, K=5, I=384, seed=4)


@pytest.fixture(autouse=True)
def _device_status_clean():
    yield
    assert B.device_status() == 0


def oracle_shard_rows(cfg, act, tokens, rank, n):
    """The oracle on shard `rank` of `n`: every expert's weights sliced to the intermediate
    columns [rank*I/n, (rank+1)*I/n) (rows of w1's gate and up halves, columns of w2)."""
    Is, nb = cfg.I // n, cfg.I // n // 128
    rows = torch.cat([torch.arange(rank * Is, (rank + 1) * Is), cfg.I + torch.arange(rank * Is, (rank + 1) * Is)])
    brows = torch.cat([torch.arange(rank * nb, (rank + 1) * nb), cfg.I // 128 + torch.arange(rank * nb, (rank + 1) * nb)])

    def get(e):
        w1q, w1s, w2q, w2s = oracle_expert(cfg, e)
        return w1q[rows], w1s[brows], w2q[:, rank * Is:(rank + 1) * Is], w2s[:, rank * nb:(rank + 1) * nb]

    w, ids = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    sel = torch.arange(cfg.T) if tokens is None else tokens
    a8, asc = O.quant_1x128(act.x[sel])
    return O.moe_layer(a8, asc, ids[sel], w[sel], get, round_bf16=False)


@pytest.mark.parametrize("cfg,n", [(MID, 2), (MID, 4), (ODD, 3)], ids=lambda v: getattr(v, "name", str(v)))
def test_tp_shards_match_the_oracle_and_sum_to_the_layer(cfg, n):
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    act = I.moe_activations(cfg)
    args = (act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV))
    total = torch.zeros(cfg.T, cfg.H, dtype=torch.float64)
    for rank in range(n):
        shard = layer.tp_shard(rank, n)
        assert shard.cfg.I == cfg.I // n
        out = shard.forward(*args).clone()
        assert_moe_close(out, oracle_shard_rows(cfg, act, None, rank, n))
        total += out.double().cpu()
    ref, _, _ = oracle_moe_rows(cfg, act, None)
    assert_moe_close(total, ref)


def test_tp8_shard_of_the_prefill_layer_many_tokens():
    """Tensor-parallel rank 3 of 8 on the prefill layer: 256 seeded tokens, the first and
    last token and every token of the most-loaded expert, against the oracle's shard."""
    cfg = I.PREFILL
    layer = MoELayer(cfg, DEV).load_synthetic_weights()
    shard = layer.tp_shard(3, 8)
    del layer
    act = I.moe_activations(cfg)
    out = shard.forward(act.logits.to(DEV), act.bias.to(DEV), act.x.to(DEV)).clone()
    _, ids_ref = O.biased_grouped_topk(act.logits, act.bias, cfg.K, cfg.G, cfg.TG, cfg.renorm, cfg.scale)
    tokens, _ = full_size_tokens(cfg, ids_ref, 256, seed=8, m64_tail=False)
    assert tokens.numel() >= 256
    assert_moe_close(out.cpu()[tokens], oracle_shard_rows(cfg, act, tokens, 3, 8))
