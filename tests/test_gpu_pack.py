"""hyb_pack on the GPU against the CPU oracle: bit-exact values, masks and
offsets (PATCH §2 tiles; 3BASiL §2A magnitude projection per 2:4 group;
SparseDecoding abstract: bitmask + fixed stride)."""
import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_pack_equal, case, dev

pytestmark = pytest.mark.gpu


def _pack_and_compare(orc, W, tmap, b1, b2):
    ref = orc.pack(inputs.bits(W), b1, b2, tmap)
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    assert_pack_equal(P, ref)
    return P


def test_pack_tiny_256(orc):
    tmap = inputs.tile_map_exact(16, 8, inputs.seed_of("tiny_256", "map"))
    W, tmap, _, _ = case(256, 256, 64, 64, tmap, name="tiny_256")
    _pack_and_compare(orc, W, tmap, 64, 64)


def test_pack_attn_4096(orc):
    tmap = inputs.attn_map(1024)
    W, tmap, _, _ = case(4096, 4096, 128, 128, tmap, name="attn_4096")
    _pack_and_compare(orc, W, tmap, 128, 128)


@pytest.mark.parametrize("shape", [(14336, 4096), (4096, 14336)])
@pytest.mark.parametrize("frac", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_pack_ffn_sweep(orc, shape, frac):
    n, k = shape
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of("ffn_sweep", n, k, frac))
    W, tmap, _, _ = case(n, k, 128, 128, tmap, outliers=0.01, name="ffn_sweep")
    _pack_and_compare(orc, W, tmap, 128, 128)


def test_pack_llama8b_layer(orc):
    f = inputs.chain_fraction(0)
    for role, n, k in inputs.LLAMA8B_LAYER:
        T = (n // 128) * (k // 64)
        tmap = inputs.tile_map_fraction(T, f, inputs.seed_of("llama8b_chain", 0, role, "map"))
        W, tmap, _, _ = case(n, k, 128, 64, tmap, name=f"llama8b/{role}")
        _pack_and_compare(orc, W, tmap, 128, 64)


def test_pack_llama70b_ffn(orc):
    for role, n, k in inputs.LLAMA70B_FFN:
        T = (n // 128) * (k // 128)
        tmap = np.ones(T, np.uint8)
        W, tmap, _, _ = case(n, k, 128, 128, tmap, std=0.015, name=f"llama70b/{role}")
        _pack_and_compare(orc, W, tmap, 128, 128)


@pytest.mark.parametrize("tiling", [(16, 16), (32, 32), (8, 16), (1, 128), (128, 16),
                                    (16, 8), (128, 8), (64, 24)])
def test_pack_other_tilings(orc, tiling):
    b1, b2 = tiling
    n, k = b1 * 6, b2 * 5
    T = 30
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("tilings", b1, b2))
    W, tmap, _, _ = case(n, k, b1, b2, tmap, name="tilings")
    _pack_and_compare(orc, W, tmap, b1, b2)


def test_pack_adversarial_ties(orc):
    """All-equal groups, +/-0, repeated magnitudes of opposite sign, subnormals
    and +/-inf: the lower column must win every tie, values copied bit-exactly."""
    rng = np.random.default_rng(42)
    n, k, b1, b2 = 128, 256, 64, 64
    pool = np.array([0x0000, 0x8000, 0x3F80, 0xBF80, 0x4000, 0xC000, 0x0001, 0x8001,
                     0x0002, 0x7F80, 0xFF80, 0x3F80, 0x3F80], np.uint16)
    Wbits = pool[rng.integers(0, pool.size, size=(n, k))]
    Wbits[:8, :] = 0x3F80          # all-equal groups
    Wbits[8:16, :] = 0x8000        # all negative zeros
    Wbits[16:24, 0::2] = 0x4000    # +2 / -2 alternating
    Wbits[16:24, 1::2] = 0xC000
    W = inputs.from_bits(Wbits)
    tmap = np.array([1, 1, 1, 0, 1, 1, 0, 1], np.uint8)
    _pack_and_compare(orc, W, tmap, b1, b2)


def test_pack_nan_sets_status(orc):
    n, k, b1, b2 = 128, 128, 64, 64
    W, _, _, _ = case(n, k, b1, b2, np.ones(4, np.uint8), name="nan")
    Wb = inputs.bits(W).copy()
    Wb[70, 9] = 0x7FC1  # NaN inside a 2:4 tile
    tmap = np.array([1, 0, 1, 1], np.uint8)
    ref = orc.pack(Wb, b1, b2, tmap)
    assert ref["nan_groups"] == 1
    Wd = inputs.from_bits(Wb).to(dev())
    ws = hyb.new_workspace(hyb.pack_workspace_bytes(), dev())
    P = hyb.pack(Wd, tmap, b1, b2, ws=ws, check=False)
    with pytest.raises(hyb.HybError) as ei:
        hyb.check_status(ws)
    assert ei.value.flags & hyb.STATUS_NAN
    assert hyb.check_status(ws) == 0  # cleared
    assert_pack_equal(P, ref)         # still complete and deterministic


def test_pack_bad_device_map_sets_status():
    """A device map byte other than 0/1 (sizes from a host map where that tile
    is dense): the device flags it and treats the tile as dense."""
    import ctypes
    n, k, b1, b2 = 128, 128, 64, 64
    W, _, _, _ = case(n, k, b1, b2, np.zeros(4, np.uint8), name="badmap")
    host_map = np.array([0, 1, 0, 0], np.uint8)
    nv, nm = hyb.packed_sizes(n, k, b1, b2, host_map)
    dmap = torch.tensor([2, 1, 0, 0], dtype=torch.uint8, device=dev())
    Wd = hyb._bits(W.to(dev()))
    vals = torch.empty(nv, dtype=torch.int16, device=dev())
    meta = torch.empty(max(nm, 1), dtype=torch.uint8, device=dev())
    vo = torch.empty(5, dtype=torch.int64, device=dev())
    mo = torch.empty(5, dtype=torch.int64, device=dev())
    ws = hyb.new_workspace(hyb.pack_workspace_bytes(), dev())
    P = ctypes.c_void_p
    rc = hyb.lib().hyb_pack(n, k, b1, b2, P(Wd.data_ptr()), k, P(dmap.data_ptr()),
                            P(vals.data_ptr()), P(meta.data_ptr()), P(vo.data_ptr()),
                            P(mo.data_ptr()), P(ws.data_ptr()), ws.numel(), hyb._stream())
    assert rc == hyb.HYB_OK
    with pytest.raises(hyb.HybError) as ei:
        hyb.check_status(ws)
    assert ei.value.flags & hyb.STATUS_BAD_MAP
    assert vo[-1].item() == nv and mo[-1].item() == nm
