"""hyb_spmv_noalloc -- the product for callers that cannot allocate device
memory: an engine that owns all device memory in one arena sized at start-up,
code running under CUDA-graph capture (cudaMalloc is not permitted there), a
memory pool that refuses allocations after set-up.

It must give the same result as hyb_spmv, the entry point that takes a caller
workspace, on consecutive calls that reuse its one static scratch array, and
stay within the stated tolerance of the CPU oracle.  This file is collected
last, so that a run stopping at its first failure has already run every other
test; it also passes when run alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_within, case, dev

pytestmark = pytest.mark.gpu


def _call_noalloc(P, X, Y, stream=None):
    """Straight through the C ABI (no workspace argument)."""
    s = P.struct()
    Xb = hyb._bits(X).reshape(1, -1)
    return hyb.lib().hyb_spmv_noalloc(ctypes.byref(s), ctypes.c_void_p(Xb.data_ptr()),
                                      Xb.stride(0), ctypes.c_void_p(Y.data_ptr()),
                                      Y.stride(0), hyb.HYB_F32, hyb._stream(stream))


def _status():
    flags = ctypes.c_uint32(0xFFFF)
    rc = hyb.lib().hyb_spmv_noalloc_check_status(hyb._stream(), ctypes.byref(flags))
    return rc, flags.value


@pytest.mark.parametrize("shape", [(4096, 4096, 128, 128), (4096, 14336, 128, 128),
                                   (1024, 4096, 128, 64)])
def test_noalloc_matches_workspace_entry_point(orc, shape):
    n, k, b1, b2 = shape
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("noalloc", n, k))
    W, tmap, _, _ = case(n, k, b1, b2, tmap, name="noalloc")
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    xs = [inputs.activations(1, k, inputs.seed_of("noalloc", n, k, "x", i)) for i in range(2)]
    # two calls in a row on the one scratch array, no synchronisation between
    outs = [torch.full((1, n), float("nan"), device=dev()) for _ in xs]
    for x, y in zip(xs, outs):
        assert _call_noalloc(P, x.to(dev()), y) == hyb.HYB_OK
    torch.cuda.synchronize()
    assert _status() == (hyb.HYB_OK, 0)
    ref = orc.pack(inputs.bits(W), b1, b2, tmap)
    for x, y in zip(xs, outs):
        # the workspace entry point runs the same kernel with the same split and
        # the same fixed reduction order: equal bit for bit
        y_ws = hyb.spmv(P, x.to(dev()))
        assert torch.equal(y, y_ws), f"noalloc vs hyb_spmv {n}x{k}"
        # and both within the tolerance of the oracle
        y_ref, env = orc.spmv(n, k, b1, b2, tmap, ref, inputs.bits(x))
        assert_within(y.cpu().numpy(), y_ref, env, what=f"noalloc vs oracle {n}x{k}")


def test_noalloc_under_graph_capture(orc):
    """The use it exists for: two calls captured in a CUDA graph (after one
    eager call that looked up the array's address), replayed twice."""
    n, k, b1, b2 = 4096, 4096, 128, 128
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("noalloc_graph", n, k))
    W, tmap, _, _ = case(n, k, b1, b2, tmap, name="noalloc_graph")
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    xs = [inputs.activations(1, k, inputs.seed_of("noalloc_graph", "x", i)).to(dev())
          for i in range(2)]
    ys = [torch.zeros(1, n, device=dev()) for _ in xs]
    assert _call_noalloc(P, xs[0], ys[0]) == hyb.HYB_OK  # first call: eager
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for x, y in zip(xs, ys):
            assert _call_noalloc(P, x, y, torch.cuda.current_stream()) == hyb.HYB_OK
    ref = orc.pack(inputs.bits(W), b1, b2, tmap)
    for _ in range(2):
        for y in ys:
            y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for x, y in zip(xs, ys):
            y_ref, env = orc.spmv(n, k, b1, b2, tmap, ref, inputs.bits(x.cpu()))
            assert_within(y.cpu().numpy(), y_ref, env, what="noalloc graph replay")
            assert torch.equal(y, hyb.spmv(P, x))
    del g
    assert _status() == (hyb.HYB_OK, 0)


def test_noalloc_rejects_matrices_beyond_its_scratch():
    """Too many tile-row bands for the static array: a clear error, nothing run."""
    cap = hyb.spmv_noalloc_max_scratch_bytes()
    assert cap == 1 << 20
    n, k, b1, b2 = 64 * 4500, 64, 64, 64
    tmap = np.zeros(n // b1, np.uint8)
    W = torch.zeros(n, k, dtype=torch.bfloat16, device=dev())
    P = hyb.pack(W, tmap, b1, b2)
    assert hyb.workspace_bytes(P, 1) > cap
    y = torch.full((1, n), 7.0, device=dev())
    rc = _call_noalloc(P, torch.ones(1, k, dtype=torch.bfloat16, device=dev()), y)
    assert rc == hyb.HYB_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
