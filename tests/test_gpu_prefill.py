"""hyb_spmm_prefill: the hybrid product for a block of tokens on the tcgen05
tensor cores (PATCH §2 Method: dense tiles on dense tensor-core kernels, 2:4
tiles on sparse ones), against the oracle's fp64 per-row product."""
import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_within, case, dev

pytestmark = pytest.mark.gpu


SHAPES = list(hyb.PREFILL_SHAPES)


def _check(orc, n, k, m, tmap, name, rows=None, block=None):
    W, tmap, X, _ = case(n, k, 128, 128, tmap, batch=m, name=name)
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    ws = hyb.new_workspace(hyb.lib().hyb_prefill_workspace_bytes(), dev())
    Y = hyb.spmm_prefill(P, X.to(dev()), ws=ws, block=block)
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


@pytest.mark.parametrize("block", SHAPES)
@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
@pytest.mark.parametrize("m", [64, 128, 200, 300])
def test_prefill_fractions(orc, frac, m, block):
    """Every tile dense, half and half, every tile 2:4; one token block, a
    full block, ragged second blocks; every CTA shape (one band x 128 or 256
    tokens, two bands x 240 tokens)."""
    n, k = 512, 1024
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of("prefill", frac))
    _check(orc, n, k, m, tmap, f"prefill_f{frac}", block=block)


@pytest.mark.parametrize("block", SHAPES)
@pytest.mark.parametrize("m", [1, 129, 1000])
def test_prefill_ragged_tokens(orc, m, block):
    """Token counts that leave most of a block empty (rows past m read as
    zeros and are never stored); 3 bands, so the two-band shape's last CTA
    has one."""
    n, k = 384, 768
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("prefill_ragged", m))
    _check(orc, n, k, m, tmap, "prefill_ragged", block=block)


@pytest.mark.parametrize("block", SHAPES)
def test_prefill_4096_tokens(orc, block):
    """The long end of prefill: 4096 tokens on a small weight, every output
    checked."""
    n, k, m = 256, 1024, 4096
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("prefill_4096"))
    _check(orc, n, k, m, tmap, "prefill_4096", block=block)


@pytest.mark.parametrize("frac", [0.0, 0.5, 1.0])
def test_prefill_shapes_agree(frac):
    """Every CTA shape adds the same products in the same order:
    bit-identical Y (the documented contract of the choice)."""
    n, k, m = 384, 1536, 700
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of("prefill_blocks", frac))
    W, tmap, X, _ = case(n, k, 128, 128, tmap, batch=m, name="prefill_blocks")
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    Xd = X.to(dev())
    Ys = [hyb.spmm_prefill(P, Xd, block=b) for b in SHAPES] + [hyb.spmm_prefill(P, Xd)]
    torch.cuda.synchronize()
    for Y in Ys[1:]:
        assert torch.equal(Ys[0], Y)


def test_prefill_block_choice():
    """The CTA shape with the fewest modelled bytes per SM: short prompts one
    band x 128 tokens, long ones two bands x 240 tokens (one wave of 144 CTAs
    for the 4096-row FFN at 2048 tokens on 148 SMs) or x 208 tokens (the
    14336-row FFN at 2048 tokens: as many waves as 240, fewer bytes each)."""
    sms = torch.cuda.get_device_properties(dev()).multi_processor_count
    for n, m in ((128, 16), (4096, 512), (4096, 2048), (14336, 2048), (384, 700)):
        assert hyb.prefill_block_shape(n, m) in SHAPES
    assert hyb.prefill_block_shape(128, 4096)[0] == 128  # one band: no two-band CTA
    if sms == 148:
        assert hyb.prefill_block_shape(4096, 512) == (128, 128)
        assert hyb.prefill_block_shape(4096, 2048) == (256, 240)
        assert hyb.prefill_block_shape(14336, 2048) == (256, 208)  # 560 CTAs, 4 waves
    with pytest.raises(hyb.HybError):
        hyb.prefill_block_shape(0, 16)


@pytest.mark.parametrize("frac,m", [(0.0, 512), (0.5, 512), (1.0, 512), (0.5, 2048)])
def test_prefill_ffn_full_size(orc, frac, m):
    """The 4096 x 14336 down projection at 512 tokens (128-token blocks) and
    2048 tokens (two bands x 240 tokens, the bench's prefill case): sampled
    rows (every token) against the oracle."""
    n, k = 4096, 14336
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


@pytest.mark.parametrize("block", SHAPES)
def test_prefill_strided_x_and_y(orc, block):
    """X and Y as views with row strides above k and n (ldx, ldy): the same
    values as contiguous buffers, and Y's padding columns untouched."""
    n, k, m = 384, 768, 300
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("prefill_strided"))
    W, tmap, X, _ = case(n, k, 128, 128, tmap, batch=m, name="prefill_strided")
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    Xbig = torch.zeros(m, k + 64, dtype=torch.bfloat16, device=dev())
    Xbig[:, :k] = X.to(dev())
    Ybig = torch.full((m, n + 32), -7.0, dtype=torch.float32, device=dev())
    hyb.spmm_prefill(P, Xbig[:, :k], Y=Ybig[:, :n], block=block)
    Y0 = hyb.spmm_prefill(P, X.to(dev()), block=block)
    torch.cuda.synchronize()
    assert torch.equal(Ybig[:, :n], Y0)
    assert bool((Ybig[:, n:] == -7.0).all())


@pytest.mark.parametrize("block", SHAPES)
@pytest.mark.parametrize("field", ["val_off", "meta_off"])
def test_prefill_bad_offsets_are_flagged(block, field):
    """Corrupted offsets (past the value or mask buffer) of a dense and a 2:4
    tile are not copied and are reported through the status word; the launch
    completes and nothing is read out of bounds."""
    n, k, m = 384, 1024, 200
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("prefill_bad"))
    W = inputs.weight(n, k, 0.02, inputs.seed_of("prefill_bad", "W")).to(dev())
    P = hyb.pack(W, tmap, 128, 128)
    t_dense = int(np.flatnonzero(tmap == 0)[0])
    t_sparse = int(np.flatnonzero(tmap == 1)[-1])
    if field == "val_off":
        P.val_off[t_dense] = P.n_vals + 128 * 128
        P.val_off[t_sparse] = P.n_vals + 64 * 128
    else:  # only a 2:4 tile reads masks
        P.meta_off[t_sparse] = P.n_meta + 4096
    ws = hyb.new_workspace(hyb.lib().hyb_prefill_workspace_bytes(), dev())
    X = torch.ones(m, k, dtype=torch.bfloat16, device=dev())
    hyb.spmm_prefill(P, X, ws=ws, block=block)
    with pytest.raises(hyb.HybError) as e:
        hyb.check_status(ws)
    assert e.value.status == hyb.HYB_ERR_DEVICE_CHECK
    assert e.value.flags & hyb.STATUS_BAD_MAP
    assert not e.value.flags & hyb.STATUS_TIMEOUT
    hyb.check_status(ws)  # cleared


@pytest.mark.parametrize("block", [(128, 64), (256, 256), (256, 0), (0, 128)])
def test_prefill_rejects_bad_block(block):
    """A CTA shape the kernel is not built for: an argument error."""
    W = torch.zeros(128, 128, dtype=torch.bfloat16, device=dev())
    P = hyb.pack(W, np.zeros(1, np.uint8), 128, 128)
    X = torch.zeros(4, 128, dtype=torch.bfloat16, device=dev())
    with pytest.raises(hyb.HybError) as e:
        hyb.spmm_prefill(P, X, block=block)
    assert e.value.status == hyb.HYB_ERR_INVALID_ARG


def test_prefill_rejects_other_tilings():
    """Only 128 x 128 tiles run on this path: a clear error, nothing queued."""
    W = torch.zeros(256, 512, dtype=torch.bfloat16, device=dev())
    P = hyb.pack(W, np.zeros((256 // 64) * (512 // 64), np.uint8), 64, 64)
    X = torch.zeros(16, 512, dtype=torch.bfloat16, device=dev())
    with pytest.raises(hyb.HybError) as e:
        hyb.spmm_prefill(P, X)
    assert e.value.status == hyb.HYB_ERR_UNSUPPORTED
