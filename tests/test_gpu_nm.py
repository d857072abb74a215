"""Tiles that are dense or N:M sparse for a general N:M (hyb_pack_nm,
hyb_spmm_skinny_nm) against the oracle's N:M routines.

PATCH, "Future direction": the tile-level scheme extends to other N:M patterns
such as 4:8; SparseDecoding (authors' abstract): N:M with bitmask indexing and
a fixed stride.  Pack: bit-exact.  Product: |y - y_ref| <= 2e-3 (|W_hat| |x|)
per output, fp32 output; bf16 output within 1 ulp of the fp32 output's
rounding."""
import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_within, bf16_within_one_ulp, dev

pytestmark = pytest.mark.gpu

NM = [(4, 8), (2, 8), (6, 8), (1, 4), (3, 4), (2, 4), (4, 16), (8, 16)]


def _packed_host(P):
    return dict(vals=P.vals.cpu().numpy().view(np.uint16), meta=P.meta.cpu().numpy()[:P.n_meta],
                val_off=P.val_off.cpu().numpy(), meta_off=P.meta_off.cpu().numpy())


def _tie_heavy(n, k, seed):
    g = torch.Generator().manual_seed(seed)
    v = torch.randint(-3, 4, (n, k), generator=g).to(torch.float32)
    return v.to(torch.bfloat16)


def _check_pack(orc, W, tmap, b1, b2, nk, m):
    P = hyb.pack_nm(W.to(dev()), tmap, b1, b2, nk, m)
    ref = orc.pack_nm(inputs.bits(W), b1, b2, tmap, nk, m)
    got = _packed_host(P)
    for key in ("val_off", "meta_off", "vals", "meta"):
        assert np.array_equal(got[key], ref[key]), (key, nk, m)
    return P, ref


@pytest.mark.parametrize("nk,m", NM)
@pytest.mark.parametrize("shape", [(256, 512, 64, 64), (384, 256, 128, 128), (128, 1024, 64, 128)])
def test_pack_nm_bit_exact(orc, nk, m, shape):
    n, k, b1, b2 = shape
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("nm_pack", n, k, nk, m))
    # normal weights with outliers, and small integers (many ties, signed zeros)
    W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_pack", n, k, "W"), outliers=0.01)
    _check_pack(orc, W, tmap, b1, b2, nk, m)
    _check_pack(orc, _tie_heavy(n, k, 17), tmap, b1, b2, nk, m)


def test_pack_nm_2of4_is_hyb_pack():
    n, k, b1, b2 = 512, 512, 128, 64
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("nm_24", n, k))
    W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_24", "W")).to(dev())
    a = _packed_host(hyb.pack(W, tmap, b1, b2, plan=False))
    b = _packed_host(hyb.pack_nm(W, tmap, b1, b2, 2, 4))
    for key in ("val_off", "meta_off", "vals", "meta"):
        assert np.array_equal(a[key], b[key]), key


@pytest.mark.parametrize("nk,m", NM)
@pytest.mark.parametrize("batch", [1, 3, 8, 16])
def test_spmm_nm_parity(orc, nk, m, batch):
    n, k, b1, b2 = 640, 1024, 128, 64
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("nm_spmm", nk, m))
    W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_spmm", "W"), outliers=0.01)
    X = inputs.activations(batch, k, inputs.seed_of("nm_spmm", "X", batch))
    P, ref = _check_pack(orc, W, tmap, b1, b2, nk, m)
    Y = hyb.spmm_skinny_nm(P, X.to(dev()), nk, m)
    torch.cuda.synchronize()
    y_ref, env = orc.spmv_nm(n, k, b1, b2, nk, m, tmap, ref, inputs.bits(X))
    assert_within(Y.cpu().numpy(), y_ref, env, what=f"{nk}:{m} b={batch}")
    Yb = hyb.spmm_skinny_nm(P, X.to(dev()), nk, m, ydt=hyb.HYB_BF16)
    bf16_within_one_ulp(Yb, Y)
    # deterministic: a second run is bit-identical
    Y2 = hyb.spmm_skinny_nm(P, X.to(dev()), nk, m)
    assert torch.equal(Y, Y2)


@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_spmm_nm_full_size_4of8(orc, frac):
    """4096 x 14336 (the down projection), 128 x 128 tiles, 4:8, batch 2."""
    n, k, b1, b2 = 4096, 14336, 128, 128
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of("nm_full", frac))
    W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_full", "W"), outliers=0.01)
    X = inputs.activations(2, k, inputs.seed_of("nm_full", "X"))
    P, ref = _check_pack(orc, W, tmap, b1, b2, 4, 8)
    Y = hyb.spmm_skinny_nm(P, X.to(dev()), 4, 8)
    torch.cuda.synchronize()
    y_ref, env = orc.spmv_nm(n, k, b1, b2, 4, 8, tmap, ref, inputs.bits(X))
    assert_within(Y.cpu().numpy(), y_ref, env, what=f"4:8 full f={frac}")


def test_spmm_nm_strided_operands(orc):
    n, k, b1, b2 = 512, 512, 64, 64
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("nm_strided"))
    W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_strided", "W"))
    X = inputs.activations(3, k, inputs.seed_of("nm_strided", "X"))
    P, ref = _check_pack(orc, W, tmap, b1, b2, 4, 8)
    Xs = torch.zeros(3, k + 40, dtype=torch.bfloat16, device=dev())
    Xs[:, 8:8 + k] = X.to(dev())
    Ys = torch.full((3, n + 24), 7.0, device=dev())
    hyb.spmm_skinny_nm(P, Xs[:, 8:8 + k], 4, 8, Y=Ys[:, 4:4 + n])
    torch.cuda.synchronize()
    y_ref, env = orc.spmv_nm(n, k, b1, b2, 4, 8, tmap, ref, inputs.bits(X))
    assert_within(Ys[:, 4:4 + n].cpu().numpy(), y_ref, env, what="4:8 strided")
    assert bool((Ys[:, :4] == 7.0).all()) and bool((Ys[:, 4 + n:] == 7.0).all())


_FRESH = """
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
from sparse_weight_b200 import hyb, inputs
n, k, b1, b2, batch = 512, 512, 64, 64, 3
tmap = inputs.tile_map_fraction((n // b1) * (k // b2), 0.5, inputs.seed_of("nm_fresh"))
W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_fresh", "W")).to("cuda")
X = inputs.activations(batch, k, inputs.seed_of("nm_fresh", "X")).to("cuda")
P = hyb.pack_nm(W, tmap, b1, b2, 4, 8)
Y = hyb.spmm_skinny_nm(P, X, 4, 8)
torch.cuda.synchronize()
np.save(sys.argv[2], Y.cpu().numpy())
"""


def test_spmm_nm_4of8_first_product_of_a_process(orc, tmp_path):
    """The 4:8 selector table in shared memory is whole in every CTA: with
    64-row tiles the producer warp's threads own table entries too.  Run as
    the first product of a fresh process (no earlier kernel has left a table
    in shared memory), a 64 x 64-tile 4:8 product matches the oracle."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = str(tmp_path / "y.npy")
    subprocess.run([sys.executable, "-c", _FRESH, root, out], check=True, timeout=300)
    n, k, b1, b2, batch = 512, 512, 64, 64, 3
    tmap = inputs.tile_map_fraction((n // b1) * (k // b2), 0.5, inputs.seed_of("nm_fresh"))
    W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_fresh", "W"))
    X = inputs.activations(batch, k, inputs.seed_of("nm_fresh", "X"))
    ref = orc.pack_nm(inputs.bits(W), b1, b2, tmap, 4, 8)
    y_ref, env = orc.spmv_nm(n, k, b1, b2, 4, 8, tmap, ref, inputs.bits(X))
    assert_within(np.load(out), y_ref, env, what="4:8 64x64 fresh process")


@pytest.mark.parametrize("nk,m", [(4, 8), (2, 8)])
def test_spmm_nm_bad_offsets_are_flagged(nk, m):
    """A corrupted offset (past the value buffer) is skipped and reported
    through the status word; nothing is read out of bounds.  4:8 runs the
    streaming kernel (whose producer checks every stage's byte ranges), 2:8
    the one-warp-per-row kernel."""
    n, k, b1, b2 = 256, 256, 64, 64
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("nm_bad"))
    W = inputs.weight(n, k, 0.02, inputs.seed_of("nm_bad", "W")).to(dev())
    P = hyb.pack_nm(W, tmap, b1, b2, nk, m)
    P.val_off[3] = P.n_vals + 4096  # past the end of the values
    P.plan, P.plan_ctas = None, 0  # the kernel reads the (corrupted) offsets itself
    ws = hyb.new_workspace(hyb.workspace_bytes(P, 1), dev())
    hyb.spmm_skinny_nm(P, torch.ones(1, k, dtype=torch.bfloat16, device=dev()), nk, m, ws=ws)
    with pytest.raises(hyb.HybError) as e:
        hyb.check_status(ws)
    assert e.value.status == hyb.HYB_ERR_DEVICE_CHECK
    assert e.value.flags & hyb.STATUS_BAD_MAP
    hyb.check_status(ws)  # cleared
