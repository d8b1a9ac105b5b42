"""Per-head sharding through the CUDA path (needs a B200): the shards of one
layer that the ranks of a multi-GPU run would take, run one after another on
one GPU, give the whole layer's kept lists and output bit for bit (every
(batch, head) is independent, so no exchange is needed)."""
import pytest
import torch

from block_sparse_attention_row_b200 import check_device_error, head_range, head_shard, sparse_attn_fwd, sparse_attn_mask

from _gpu_cases import workload

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,world", [("mid", 3), ("sweep", 8), ("tiny", 2)])
def test_head_shards_reproduce_the_whole_layer(name, world):
    cfg, (Q, K, V), _ = workload(name)
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, cfg.k, cfg.p)
    O = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, cfg.bk)
    BH = cfg.B * cfg.H
    flat = lambda t: t.reshape((BH,) + tuple(t.shape[2:]))
    for r in range(world):
        lo, hi = head_range(BH, world, r)
        Qs, Ks, Vs = (head_shard(x, world, r) for x in (Q, K, V))
        ms = sparse_attn_mask(Qs, Ks, cfg.bq, cfg.bk, cfg.k, cfg.p)
        Os = sparse_attn_fwd(Qs, Ks, Vs, ms["cnt"], ms["idx"], cfg.bq, cfg.bk)
        assert torch.equal(ms["cnt"][0], flat(m["cnt"])[lo:hi])
        kept = torch.arange(cfg.n_k, device=Q.device) < ms["cnt"][0][..., None]
        assert torch.equal(ms["idx"][0][kept], flat(m["idx"])[lo:hi][kept])
        assert torch.equal(Os[0], flat(O)[lo:hi])
    check_device_error(Q.device)
