"""hyb_gemv_dense (the dense baseline) and hyb_lowrank_add against the oracle."""
import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_within, bf16_within_one_ulp, dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(4096, 4096), (1024, 4096), (4096, 14336), (14336, 4096),
                                   (192, 320), (100, 48), (7, 32)])
@pytest.mark.parametrize("batch", [1, 4, 16])
def test_gemv_dense(orc, shape, batch):
    n, k = shape
    W = inputs.weight(n, k, 0.02, inputs.seed_of("dense", n, k))
    X = inputs.activations(batch, k, inputs.seed_of("dense", n, k, "X"))
    Y = hyb.gemv_dense(W.to(dev()), X.to(dev()))
    torch.cuda.synchronize()
    if n * k <= 4096 * 4096:
        y_ref, env = orc.matvec(inputs.bits(W), inputs.bits(X))
        assert_within(Y.cpu().numpy(), y_ref, env, what=f"dense {n}x{k}")
    else:
        rows = np.unique(np.concatenate([[0, n - 1],
                                         np.random.default_rng(1).integers(0, n, 200)]))
        y_ref, env = orc.matvec(inputs.bits(W)[rows], inputs.bits(X))
        assert_within(Y.cpu().numpy()[:, rows], y_ref, env, what=f"dense {n}x{k}")
    Yb = hyb.gemv_dense(W.to(dev()), X.to(dev()), ydt=hyb.HYB_BF16)
    bf16_within_one_ulp(Yb, Y)


@pytest.mark.parametrize("batch", [1, 3, 16])
@pytest.mark.parametrize("rank", [8, 64, 128, 256])
def test_lowrank_add(orc, batch, rank):
    n, k = 1024, 2048
    U, V = inputs.lowrank(n, k, rank, 0.01, inputs.seed_of("lr", rank))
    X = inputs.activations(batch, k, inputs.seed_of("lr", "X", batch))
    Y0 = torch.randn(batch, n, generator=torch.Generator().manual_seed(3))
    Y = Y0.to(dev()).clone()
    hyb.lowrank_add(U.to(dev()), V.to(dev()), X.to(dev()), Y)
    zeros = np.zeros((n, k), np.uint16)
    y_ref, env = orc.matvec(zeros, inputs.bits(X), inputs.bits(U), inputs.bits(V))
    got = Y.cpu().numpy().astype(np.float64) - Y0.numpy().astype(np.float64)
    # the in-place add rounds once more in fp32: allow that rounding on top
    env2 = env + np.abs(Y0.numpy()) * 2 ** -23 / 2e-3
    assert_within(got, y_ref, env2, what=f"lowrank r={rank} b={batch}")
