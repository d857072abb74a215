"""hyb_spmm_prefill: the hybrid product for a block of tokens on the tcgen05
tensor cores (PATCH §2 Method: dense tiles on dense tensor-core kernels, 2:4
tiles on sparse ones), against the oracle's fp64 per-row product."""
import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_within, case, dev

pytestmark = pytest.mark.gpu


def _check(orc, n, k, m, tmap, name, rows=None):
    W, tmap, X, _ = case(n, k, 128, 128, tmap, batch=m, name=name)
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    ws = hyb.new_workspace(hyb.lib().hyb_prefill_workspace_bytes(), dev())
    Y = hyb.spmm_prefill(P, X.to(dev()), ws=ws)
    torch.cuda.synchronize()
    assert hyb.check_status(ws) == 0
    Yh = Y.cpu().numpy()
    if rows is None:
        ref = orc.pack(inputs.bits(W), 128, 128, tmap)
        y_ref, env = orc.spmv(n, k, 128, 128, tmap, ref, inputs.bits(X))
        assert_within(Yh, y_ref, env, what=f"prefill {n}x{k} m={m}")
    else:
        y_ref, env = orc.rows(inputs.bits(W), 128, 128, tmap, inputs.bits(X), rows)
        assert_within(Yh[:, rows], y_ref, env, what=f"prefill {n}x{k} m={m} sampled")
    return P, X, Y


@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
@pytest.mark.parametrize("m", [64, 128, 200])
def test_prefill_fractions(orc, frac, m):
    """Every tile dense, half and half, every tile 2:4; one token block, a
    full block, a ragged second block."""
    n, k = 512, 1024
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of("prefill", frac))
    _check(orc, n, k, m, tmap, f"prefill_f{frac}")


@pytest.mark.parametrize("m", [1, 129, 1000])
def test_prefill_ragged_tokens(orc, m):
    """Token counts that leave most of a block empty (rows past m read as
    zeros and are never stored)."""
    n, k = 384, 768
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("prefill_ragged", m))
    _check(orc, n, k, m, tmap, "prefill_ragged")


def test_prefill_4096_tokens(orc):
    """The long end of prefill: 4096 tokens (32 token blocks) on a small
    weight, every output checked."""
    n, k, m = 256, 1024, 4096
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("prefill_4096"))
    _check(orc, n, k, m, tmap, "prefill_4096")


@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_prefill_ffn_full_size(orc, frac):
    """The 4096 x 14336 down projection at 512 tokens: sampled rows (every
    token) against the oracle."""
    n, k, m = 4096, 14336, 512
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of("prefill_ffn", frac))
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 2047, 4095],
                                     rng.integers(0, n, 10)])).astype(np.int64)
    _check(orc, n, k, m, tmap, "prefill_ffn", rows=rows)


def test_prefill_matches_the_dense_path(orc):
    """An all-dense map through the tensor cores equals the bf16 weights times
    X within the tolerance, and the same W with every tile 2:4 equals the
    magnitude-pruned weights (expansion puts each kept pair in place)."""
    n, k, m = 256, 512, 96
    T = (n // 128) * (k // 128)
    for frac in (0.0, 1.0):
        tmap = np.full(T, 1 if frac else 0, np.uint8)
        P, X, Y = _check(orc, n, k, m, tmap, "prefill_eq")
        # deterministic: a second call is bit-identical
        Y2 = hyb.spmm_prefill(P, X.to(dev()))
        torch.cuda.synchronize()
        assert torch.equal(Y, Y2)


def test_prefill_rejects_other_tilings():
    """Only 128 x 128 tiles run on this path: a clear error, nothing queued."""
    W = torch.zeros(256, 512, dtype=torch.bfloat16, device=dev())
    P = hyb.pack(W, np.zeros((256 // 64) * (512 // 64), np.uint8), 64, 64)
    X = torch.zeros(16, 512, dtype=torch.bfloat16, device=dev())
    with pytest.raises(hyb.HybError) as e:
        hyb.spmm_prefill(P, X)
    assert e.value.status == hyb.HYB_ERR_UNSUPPORTED
