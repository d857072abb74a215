"""Products launched with HYB_LAUNCH_OVERLAP_PREV (programmatic dependent
launch: the product's CTAs may start, and request weight bytes, while the
kernel queued before it is still running).

The flag changes when the work starts, never what it computes, so every
result here must equal, bit for bit, the same sequence launched without the
flag -- the product is deterministic (fixed split, CTA-ordered sums).  The
sequences are chains in which each product's X is the bf16 output of the
product queued just before it, all products sharing one workspace (the band
tickets and split slots that the preceding product also uses): exactly the
accesses that must wait for the preceding grid.  The first layer is also
checked against the oracle."""
import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_within, bf16_within_one_ulp, dev

pytestmark = pytest.mark.gpu


def _layers(shapes, b1, b2, frac, name, rank=0):
    """Seeded packed layers; weights N(0, 1/sqrt(k)) keep the activations O(1)."""
    mats, dense, lrs, host = [], [], [], []
    for l, (n, k) in enumerate(shapes):
        T = (n // b1) * (k // b2)
        tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of(name, l, "map"))
        W = inputs.weight(n, k, 1.0 / np.sqrt(k), inputs.seed_of(name, l, "W"))
        Wd = W.to(dev())
        mats.append(hyb.pack(Wd, tmap, b1, b2))
        dense.append(Wd)
        if rank:
            U, V = inputs.lowrank(n, k, rank, 0.01, inputs.seed_of(name, l, "LR"))
            lrs.append((U.to(dev()), V.to(dev())))
            host.append((W, tmap, U, V))
        else:
            lrs.append(None)
            host.append((W, tmap, None, None))
    return mats, dense, lrs, host


def _run_chain(step, shapes, x0, flags, graph, between):
    """ys[l] = layer l applied to ys[l-1] (x0 for l = 0), bf16 outputs."""
    batch = x0.shape[0]
    ys = [torch.full((batch, n), float("nan"), dtype=torch.bfloat16, device=dev())
          for n, _ in shapes]
    # staging buffers for the variant with a torch kernel between products
    xs = [torch.empty(batch, n, dtype=torch.bfloat16, device=dev()) for n, _ in shapes]

    def run():
        x = x0
        for l in range(len(shapes)):
            step(l, x, ys[l], flags)
            if between:
                torch.mul(ys[l], 1.0, out=xs[l])  # a non-library kernel writes the next X
                x = xs[l]
            else:
                x = ys[l]

    if graph:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            run()  # warm-up outside the capture
        torch.cuda.synchronize()
        for y in ys:
            y.fill_(float("nan"))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            run()
        g.replay()
        torch.cuda.synchronize()
        del g
    else:
        run()
        torch.cuda.synchronize()
    return [y.clone() for y in ys]


CHAINS = {
    # down-projection feeding square layers: a long product, then short ones
    "ffn": ([(14336, 4096), (4096, 14336), (4096, 4096), (4096, 4096)], 128, 128),
    "attn": ([(4096, 4096)] * 6, 128, 64),
    # few tiles: fewer CTAs than SMs, so the next product's CTAs find idle SMs
    "small": ([(512, 512)] * 6, 64, 64),
}


@pytest.mark.parametrize("chain,batch,frac,rank,graph,between", [
    ("ffn", 1, 0.5, 0, False, False),
    ("ffn", 1, 0.5, 0, True, False),
    ("ffn", 8, 0.5, 0, True, False),
    ("attn", 4, 0.25, 0, False, False),
    ("attn", 16, 0.75, 0, True, False),
    ("attn", 1, 0.5, 64, True, False),
    ("small", 1, 0.5, 0, True, False),
    ("small", 2, 1.0, 0, False, True),
    ("ffn", 1, 0.0, 0, True, True),
])
def test_overlapped_chain_equals_plain_chain(orc, chain, batch, frac, rank, graph, between):
    shapes, b1, b2 = CHAINS[chain]
    name = f"overlap_{chain}_{frac}_{rank}"
    mats, _, lrs, host = _layers(shapes, b1, b2, frac, name, rank)
    ws = hyb.new_workspace(max(hyb.workspace_bytes(m, batch, rank) for m in mats), dev())
    x0 = inputs.activations(batch, shapes[0][1], inputs.seed_of(name, "x0", batch)).to(dev())

    def step(l, x, y, flags):
        hyb.spmm_skinny(mats[l], x, Y=y, ydt=hyb.HYB_BF16, lowrank=lrs[l], ws=ws, flags=flags)

    plain = _run_chain(step, shapes, x0, 0, graph, between)
    over = _run_chain(step, shapes, x0, hyb.LAUNCH_OVERLAP_PREV, graph, between)
    for l, (a, b) in enumerate(zip(plain, over)):
        assert not torch.isnan(a.float()).any(), f"layer {l}: output not written"
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"layer {l} differs"

    # layer 0 against the oracle (fp32 output; bf16 output is its rounding)
    y32 = hyb.spmm_skinny(mats[0], x0, lowrank=lrs[0], ws=ws)
    torch.cuda.synchronize()
    bf16_within_one_ulp(over[0], y32)
    n, k = shapes[0]
    W, tmap, U, V = host[0]
    ref = orc.pack(inputs.bits(W), b1, b2, tmap)
    y_ref, env = orc.spmv(n, k, b1, b2, tmap, ref, inputs.bits(x0.cpu()),
                          None if U is None else inputs.bits(U),
                          None if V is None else inputs.bits(V))
    assert_within(y32.cpu().numpy(), y_ref, env, what=f"{chain} layer 0")


@pytest.mark.parametrize("batch,graph", [(1, True), (4, False), (16, True)])
def test_overlapped_dense_chain_equals_plain_chain(batch, graph):
    shapes = [(4096, 4096)] * 4
    _, dense, _, _ = _layers(shapes, 128, 128, 0.0, "overlap_dense")
    ws = hyb.new_workspace(hyb.dense_workspace_bytes(4096, 4096, batch), dev())
    x0 = inputs.activations(batch, 4096, inputs.seed_of("overlap_dense", "x0", batch)).to(dev())

    def step(l, x, y, flags):
        hyb.gemv_dense(dense[l], x, Y=y, ydt=hyb.HYB_BF16, ws=ws, flags=flags)

    plain = _run_chain(step, shapes, x0, 0, graph, False)
    over = _run_chain(step, shapes, x0, hyb.LAUNCH_OVERLAP_PREV, graph, False)
    for l, (a, b) in enumerate(zip(plain, over)):
        assert not torch.isnan(a.float()).any(), f"layer {l}: output not written"
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"layer {l} differs"
    # (the fp32 product itself is checked against the oracle in the dense tests)
    y32 = hyb.gemv_dense(dense[0], x0, ws=ws)
    torch.cuda.synchronize()
    bf16_within_one_ulp(over[0], y32)
