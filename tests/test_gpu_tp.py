"""Row-sharded (tensor-parallel) decode on one GPU: every rank's shard of a
packed matrix (views of its bands, rebased offsets, its own split) run by the
library's product, the rows put together and checked against the oracle.
The collective itself is tested with gloo ranks on CPU (test_dist_cpu.py)."""
import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs, tp
from gpu_cases import assert_within, case, dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [1, 2, 3, 5])
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_row_shards_cover_the_product(orc, world, batch):
    n, k, b1, b2 = 1280, 2048, 128, 128
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("tp_gpu", n, k))
    W, tmap, X, _ = case(n, k, b1, b2, tmap, batch=batch, name="tp_gpu")
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    Xd = X.to(dev())
    Y = torch.full((batch, n), float("nan"), device=dev())
    covered = np.zeros(n, bool)
    for r in range(world):
        sh = tp.RowShard(P, r, world)
        lo, hi = sh.rows[r]
        assert not covered[lo:hi].any()
        covered[lo:hi] = True
        if sh.local is not None:
            Y[:, lo:hi] = hyb.spmm_skinny(sh.local, Xd)
    assert covered.all()
    torch.cuda.synchronize()
    ref = orc.pack(inputs.bits(W), b1, b2, tmap)
    y_ref, env = orc.spmv(n, k, b1, b2, tmap, ref, inputs.bits(X))
    assert_within(Y.cpu().numpy(), y_ref, env, what=f"row shards world={world} b={batch}")


def test_single_rank_apply_equals_the_product(orc):
    """World 1 through RowShard.apply (no collective) is the unsharded product."""
    n, k, b1, b2 = 1024, 1024, 128, 128
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("tp_one"))
    W, tmap, X, _ = case(n, k, b1, b2, tmap, batch=2, name="tp_one")
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    Y = tp.RowShard(P, 0, 1).apply(X.to(dev()))
    torch.cuda.synchronize()
    assert torch.equal(Y, hyb.spmm_skinny(P, X.to(dev())))
