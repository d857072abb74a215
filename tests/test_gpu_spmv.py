"""hyb_spmv / hyb_spmm_skinny on the GPU against the fp64 CPU oracle.

Bound (spec tolerance, fp32 accumulation of bf16 products):
|y - y_ref|_i <= 2e-3 * (|W_hat| |x| + |U| (|V|^T |x|))_i, per output."""
import numpy as np
import pytest
import torch

from sparse_weight_b200 import hyb, inputs
from gpu_cases import assert_within, bf16_within_one_ulp, case, dev

pytestmark = pytest.mark.gpu


def _full_check(orc, n, k, b1, b2, tmap, batch, name, rank=0, ydt_bf16=True):
    W, tmap, X, UV = case(n, k, b1, b2, tmap, batch=batch, name=name, rank=rank)
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    Xd = X.to(dev())
    lr = tuple(t.to(dev()) for t in UV) if UV else None
    Y = hyb.spmm_skinny(P, Xd, lowrank=lr)
    torch.cuda.synchronize()
    ref = orc.pack(inputs.bits(W), b1, b2, tmap)
    U = inputs.bits(UV[0]) if UV else None
    V = inputs.bits(UV[1]) if UV else None
    y_ref, env = orc.spmv(n, k, b1, b2, tmap, ref, inputs.bits(X), U, V)
    assert_within(Y.cpu().numpy(), y_ref, env, what=f"{name} {n}x{k} b={batch}")
    if ydt_bf16:
        Yb = hyb.spmm_skinny(P, Xd, ydt=hyb.HYB_BF16, lowrank=lr)
        bf16_within_one_ulp(Yb, Y)
    return P, Xd, Y


def test_tiny_256(orc):
    tmap = inputs.tile_map_exact(16, 8, inputs.seed_of("tiny_256", "map"))
    _full_check(orc, 256, 256, 64, 64, tmap, 1, "tiny_256")


def test_attn_4096(orc):
    _full_check(orc, 4096, 4096, 128, 128, inputs.attn_map(1024), 1, "attn_4096")


def test_spmv_entry_point_batch1(orc):
    """hyb_spmv (batch-1 entry point) equals hyb_spmm_skinny at batch 1."""
    tmap = inputs.attn_map(1024)
    W, tmap, X, _ = case(4096, 4096, 128, 128, tmap, name="attn_4096")
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    y1 = hyb.spmv(P, X.to(dev()).view(-1))
    y2 = hyb.spmm_skinny(P, X.to(dev()))
    assert torch.equal(y1, y2)


@pytest.mark.parametrize("tiling", [(128, 128), (128, 64), (64, 64), (64, 128)])
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8, 13, 16])
def test_multi_tile_ragged(orc, tiling, batch):
    """Shapes that span several tiles and bands, with byte splits that end
    mid-band: every batch specialisation (and non-power-of-2 batches)."""
    b1, b2 = tiling
    n, k = b1 * 5, b2 * 11
    T = 55
    tmap = inputs.tile_map_bernoulli(T, 0.4, inputs.seed_of("ragged", b1, b2))
    _full_check(orc, n, k, b1, b2, tmap, batch, f"ragged{b1}x{b2}")


@pytest.mark.parametrize("tiling", [(128, 128), (128, 64), (64, 64), (64, 128)])
@pytest.mark.parametrize("batch", [1, 2, 3, 4, 5, 8, 13, 16])
@pytest.mark.parametrize("tpr", [7, 37])
def test_rows_ragged(orc, tiling, batch, tpr):
    """2560 output rows with 7 or 37 tiles per band: the byte split puts CTA
    boundaries mid-band and mid-window (37 tiles span two offset windows)."""
    b1, b2 = tiling
    n, k = 2560, b2 * tpr
    T = (n // b1) * tpr
    tmap = inputs.tile_map_bernoulli(T, 0.4, inputs.seed_of("rows", b1, b2, tpr))
    _full_check(orc, n, k, b1, b2, tmap, batch, f"rows{b1}x{b2}", ydt_bf16=batch in (1, 16))


@pytest.mark.parametrize("tiling", [(16, 16), (32, 32), (8, 16), (1, 128), (128, 16), (256, 64),
                                    (16, 8), (128, 8), (64, 24), (32, 40)])
@pytest.mark.parametrize("batch", [1, 3, 16])
def test_other_tilings(orc, tiling, batch):
    b1, b2 = tiling
    n, k = b1 * 6, b2 * 5
    tmap = inputs.tile_map_bernoulli(30, 0.5, inputs.seed_of("tilings", b1, b2))
    _full_check(orc, n, k, b1, b2, tmap, batch, f"tilings{b1}x{b2}")


@pytest.mark.parametrize("frac", [0.0, 1.0])
def test_degenerate_maps(orc, frac):
    """All-dense and all-2:4 maps (0 % and 50 % sparsity)."""
    T = 32 * 32
    tmap = np.full(T, int(frac), np.uint8)
    _full_check(orc, 4096, 4096, 128, 128, tmap, 4, f"degenerate{frac}")


@pytest.mark.parametrize("batch", [1, 3, 5, 16])
def test_strided_operands(orc, batch):
    """X rows with a row stride above k and a column offset, Y rows with a row
    stride above n: the result equals the contiguous call bit for bit, and the
    padding around Y is left alone (batch >= 4 fetches X by tensor copies whose
    row stride is ldx)."""
    n, k, b1, b2 = 1280, 2304, 128, 128
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("strided", n, k))
    W, tmap, X, _ = case(n, k, b1, b2, tmap, batch=batch, name="strided")
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    Xd = X.to(dev())
    big = torch.zeros(batch, k + 40, dtype=torch.bfloat16, device=dev())
    big[:, 8:8 + k] = Xd
    Xs = big[:, 8:8 + k]
    assert Xs.stride(0) == k + 40 and Xs.data_ptr() % 16 == 0
    Ybig = torch.full((batch, n + 24), 5.0, device=dev())
    Ys = Ybig[:, 4:4 + n]
    hyb.spmm_skinny(P, Xs, Y=Ys)
    Yc = hyb.spmm_skinny(P, Xd)
    torch.cuda.synchronize()
    assert torch.equal(Ys, Yc)
    assert bool((Ybig[:, :4] == 5.0).all()) and bool((Ybig[:, 4 + n:] == 5.0).all())
    y_ref, env = orc.spmv(n, k, b1, b2, tmap, orc.pack(inputs.bits(W), b1, b2, tmap),
                          inputs.bits(X))
    assert_within(Ys.cpu().numpy(), y_ref, env, what=f"strided b={batch}")


def test_single_tile(orc):
    _full_check(orc, 128, 128, 128, 128, np.array([1], np.uint8), 1, "single")
    _full_check(orc, 64, 64, 64, 64, np.array([0], np.uint8), 2, "single0")


def test_zero_input(orc):
    """x = 0 gives exactly zero output."""
    tmap = inputs.attn_map(1024)
    W, tmap, X, _ = case(4096, 4096, 128, 128, tmap, name="attn_4096")
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    y = hyb.spmv(P, torch.zeros(4096, dtype=torch.bfloat16, device=dev()))
    assert torch.count_nonzero(y).item() == 0


def test_deterministic():
    """Fixed split and fixed-order reductions: identical bits run to run."""
    tmap = inputs.attn_map(1024)
    W, tmap, X, _ = case(4096, 4096, 128, 128, tmap, batch=4, name="attn_4096")
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    Xd = X.to(dev())
    ws = hyb.new_workspace(hyb.workspace_bytes(P, 4), dev())
    first = hyb.spmm_skinny(P, Xd, ws=ws).clone()
    for _ in range(10):
        assert torch.equal(hyb.spmm_skinny(P, Xd, ws=ws), first)


def _sampled_rows(n, b1, count, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, b1 - 1, b1, n // 2, n - b1, n - 2, n - 1]
    return np.unique(np.concatenate([fixed, rng.integers(0, n, size=count)])).astype(np.int64)


@pytest.mark.parametrize("shape", [(14336, 4096), (4096, 14336)])
@pytest.mark.parametrize("frac", [0.0, 0.25, 0.5, 0.75, 1.0])
def test_ffn_sweep_full_size(orc, shape, frac):
    """Full FFN shapes with 1 % x20 outliers, the 2:4-tile fraction sweep, batch
    {1, 4, 8, 16}: sampled output rows against the oracle's per-row product."""
    n, k = shape
    T = (n // 128) * (k // 128)
    tmap = inputs.tile_map_fraction(T, frac, inputs.seed_of("ffn_sweep", n, k, frac))
    W, tmap, X, _ = case(n, k, 128, 128, tmap, batch=16, outliers=0.01, name="ffn_sweep")
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    rows = _sampled_rows(n, 128, 120, 17)
    Wb = inputs.bits(W)
    for batch in (1, 4, 8, 16):
        Xb = X[:batch]
        Y = hyb.spmm_skinny(P, Xb.to(dev())).cpu().numpy()
        y_ref, env = orc.rows(Wb, 128, 128, tmap, inputs.bits(Xb), rows)
        assert_within(Y[:, rows], y_ref, env, what=f"ffn {n}x{k} f={frac} b={batch}")


def test_llama8b_layer_full_size(orc):
    """One 32-layer-chain layer (128x64 tiles, per-layer fraction), batch 1."""
    layer = 3
    f = inputs.chain_fraction(layer)
    for role, n, k in inputs.LLAMA8B_LAYER:
        T = (n // 128) * (k // 64)
        tmap = inputs.tile_map_fraction(T, f, inputs.seed_of("llama8b_chain", layer, role, "map"))
        W, tmap, X, _ = case(n, k, 128, 64, tmap, name=f"llama8b/{layer}/{role}")
        P = hyb.pack(W.to(dev()), tmap, 128, 64)
        rows = _sampled_rows(n, 128, 64, 5)
        Y = hyb.spmv(P, X.to(dev())).cpu().numpy()
        y_ref, env = orc.rows(inputs.bits(W), 128, 64, tmap, inputs.bits(X), rows)
        assert_within(Y[:, rows], y_ref, env, what=f"llama8b {role}")


def test_llama8b_chain_every_layer(orc):
    """The 32-layer chain as the bench runs it: one weight draw per role, the
    tile map drawn per layer at that layer's fraction, all 224 matrices
    packed at full size and each product checked on sampled rows (the first
    two bands' edges, the middle, the last band's edges and six seeded random
    rows per matrix)."""
    Wr = {role: inputs.weight(n, k, 0.02, inputs.seed_of("llama8b_chain", role, "W"))
          for role, n, k in inputs.LLAMA8B_LAYER}
    Wd = {role: W.to(dev()) for role, W in Wr.items()}
    Wb = {role: inputs.bits(W) for role, W in Wr.items()}
    checked = 0
    for layer in range(32):
        f = inputs.chain_fraction(layer)
        for role, n, k in inputs.LLAMA8B_LAYER:
            T = (n // 128) * (k // 64)
            tmap = inputs.tile_map_fraction(T, f, inputs.seed_of("llama8b_chain", layer, role,
                                                                  "map"))
            X = inputs.activations(1, k, inputs.seed_of("chain_parity", layer, role))
            P = hyb.pack(Wd[role], tmap, 128, 64)
            # the realised 2:4-tile fraction is the layer's (exact count by seeded shuffle)
            assert int(tmap.sum()) == round(f * T)
            rows = _sampled_rows(n, 128, 6, layer)
            Y = hyb.spmv(P, X.to(dev())).cpu().numpy()
            y_ref, env = orc.rows(Wb[role], 128, 64, tmap, inputs.bits(X), rows)
            assert_within(Y[:, rows], y_ref, env, what=f"llama8b layer {layer} {role} f={f:.3f}")
            checked += 1
            del P
    assert checked == 224


def test_llama70b_ffn_lowrank_full_size(orc):
    """All-2:4 70B-shaped FFN plus rank-128 low-rank term, fused; batch {1,8,16}."""
    for role, n, k in inputs.LLAMA70B_FFN:
        T = (n // 128) * (k // 128)
        W, tmap, X, UV = case(n, k, 128, 128, np.ones(T, np.uint8), batch=16, std=0.015,
                              name=f"llama70b/{role}", rank=128)
        P = hyb.pack(W.to(dev()), tmap, 128, 128)
        lr = tuple(t.to(dev()) for t in UV)
        rows = _sampled_rows(n, 128, 48, 9)
        for batch in (1, 8, 16):
            Y = hyb.spmm_skinny(P, X[:batch].to(dev()), lowrank=lr).cpu().numpy()
            y_ref, env = orc.rows(inputs.bits(W), 128, 128, tmap, inputs.bits(X[:batch]),
                                  rows, inputs.bits(UV[0]), inputs.bits(UV[1]))
            assert_within(Y[:, rows], y_ref, env, what=f"70b {role} b={batch}")
        del P, W


@pytest.mark.parametrize("batch", [1, 5, 16])
def test_lowrank_fused_small(orc, batch):
    tmap = inputs.tile_map_bernoulli(40, 0.6, inputs.seed_of("lrsmall"))
    _full_check(orc, 640, 1024, 128, 128, tmap, batch, "lrsmall", rank=64)


@pytest.mark.parametrize("rank", [8, 24, 40, 128, 256])
@pytest.mark.parametrize("tiling", [(128, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("batch", [1, 3, 16])
def test_lowrank_fused_ranks(orc, rank, tiling, batch):
    """The low-rank term computed inside the streaming kernel (V^T x over
    k-slices, t summed by slices, U t by row slices, grid barriers between):
    every rank layout (16-byte chunks of a factor row that do and do not
    divide a warp), tilings whose CTA counts differ, ragged batches."""
    b1, b2 = tiling
    n, k = 10 * b1, 24 * b2
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("lrranks", b1, b2))
    _full_check(orc, n, k, b1, b2, tmap, batch, f"lrranks{rank}", rank=rank)


def test_lowrank_fused_repeated_calls(orc):
    """The fused term's grid barrier and partial buffers are left ready for
    the next call: calls in a row, alternating ranks, on one workspace."""
    n, k, b1, b2 = 1024, 2048, 128, 128
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_bernoulli(T, 0.5, inputs.seed_of("lrrep"))
    W, tmap, X, _ = case(n, k, b1, b2, tmap, batch=4, name="lrrep")
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    ws = hyb.new_workspace(hyb.workspace_bytes(P, 4, 128), dev())
    ref = orc.pack(inputs.bits(W), b1, b2, tmap)
    outs = []
    for i, rank in enumerate([128, 64, 128, 8]):
        U, V = inputs.lowrank(n, k, rank, 0.01, inputs.seed_of("lrrep", i))
        Y = hyb.spmm_skinny(P, X.to(dev()), lowrank=(U.to(dev()), V.to(dev())), ws=ws)
        outs.append((U, V, Y))
    torch.cuda.synchronize()
    assert hyb.check_status(ws) == 0
    for U, V, Y in outs:
        y_ref, env = orc.spmv(n, k, b1, b2, tmap, ref, inputs.bits(X), inputs.bits(U),
                              inputs.bits(V))
        assert_within(Y.cpu().numpy(), y_ref, env, what=f"repeated r={U.shape[1]}")


@pytest.mark.parametrize("batch", [1, 3, 8, 16])
@pytest.mark.parametrize("shape", [(1024, 2048, 128, 128), (1536, 1024, 128, 64)])
def test_gate_up_shared_lowrank(orc, batch, shape):
    """Gate and up projections of one input with one shared V (3BASiL §1:
    W ~ S + U V^T; the same x, so the same V^T x): each output within the
    oracle's tolerance of (S + U V^T) x; the gate output bit-identical to a
    separate call, the up output too where a separate up call would reduce t
    over the same split (same CTA count, or the three-kernel path of batch 8
    and 16, whose V^T x split depends on k only).  Batch <= 4 takes the fused
    path."""
    n, k, b1, b2 = shape
    T = (n // b1) * (k // b2)
    rank = 64
    Wg, tg, X, _ = case(n, k, b1, b2, inputs.tile_map_bernoulli(
        T, 0.5, inputs.seed_of("gateup", "g", n)), batch=batch, name="gateup_g")
    Wu, tu, _, _ = case(n, k, b1, b2, inputs.tile_map_bernoulli(
        T, 0.5, inputs.seed_of("gateup", "u", n)), batch=batch, name="gateup_u")
    Ug, V = inputs.lowrank(n, k, rank, 0.01, inputs.seed_of("gateup", "lr_g", n))
    Uu, _ = inputs.lowrank(n, k, rank, 0.01, inputs.seed_of("gateup", "lr_u", n))
    Pg = hyb.pack(Wg.to(dev()), tg, b1, b2)
    Pu = hyb.pack(Wu.to(dev()), tu, b1, b2)
    Xd, Ugd, Uud, Vd = X.to(dev()), Ug.to(dev()), Uu.to(dev()), V.to(dev())
    ws = hyb.new_workspace(hyb.gate_up_workspace_bytes(Pg, Pu, batch, rank), dev())
    Yg, Yu = hyb.spmm_skinny_gate_up(Pg, Pu, Xd, Ugd, Uud, Vd, ws=ws)
    # a second time on the same workspace, as a chain of layers would
    Yg2, Yu2 = hyb.spmm_skinny_gate_up(Pg, Pu, Xd, Ugd, Uud, Vd, ws=ws,
                                       flags=hyb.LAUNCH_OVERLAP_PREV)
    Yg_sep = hyb.spmm_skinny(Pg, Xd, lowrank=(Ugd, Vd))
    Yu_sep = hyb.spmm_skinny(Pu, Xd, lowrank=(Uud, Vd))
    torch.cuda.synchronize()
    assert hyb.check_status(ws) == 0
    assert torch.equal(Yg, Yg_sep)
    if batch > 4 or Pg.plan_ctas == Pu.plan_ctas:
        # t reduced over the same split as in a separate up call
        assert torch.equal(Yu, Yu_sep)
    assert torch.equal(Yg, Yg2) and torch.equal(Yu, Yu2)
    for W, tmap, U, Y, nm in ((Wg, tg, Ug, Yg, "gate"), (Wu, tu, Uu, Yu, "up")):
        ref = orc.pack(inputs.bits(W), b1, b2, tmap)
        y_ref, env = orc.spmv(n, k, b1, b2, tmap, ref, inputs.bits(X), inputs.bits(U),
                              inputs.bits(V))
        assert_within(Y.cpu().numpy(), y_ref, env, what=f"gate/up shared LR {nm} b={batch}")


def _tile_split_reference(P, G):
    """CTA c's first tile is the first t whose packed byte offset P(t)
    (2 * val_off + meta_off) satisfies P(t) * G >= c * total."""
    total, T = int(P[-1]), len(P) - 1
    return [int(np.sum(P[:T] * G < c * total)) for c in range(G)] + [T]


@pytest.mark.parametrize("shape", [(4096, 14336, 128, 128), (14336, 4096, 128, 64),
                                   (256, 256, 64, 64), (1024, 4096, 128, 64)])
def test_plan_matches_definition_and_results(orc, shape):
    """hyb_make_plan (host records handed to the kernel as launch parameters)
    gives the split the kernel would search for, and the product with and
    without the plan (or with a plan for another CTA count) is the same."""
    n, k, b1, b2 = shape
    T = (n // b1) * (k // b2)
    tmap = inputs.tile_map_fraction(T, 0.5, inputs.seed_of("plan", n, k))
    W, tmap, X, _ = case(n, k, b1, b2, tmap, name="plan")
    P = hyb.pack(W.to(dev()), tmap, b1, b2)
    plan = P.plan.numpy()
    assert not P.plan.is_cuda
    G = int(plan[0])
    assert G == P.plan_ctas and int(plan[1]) == 1
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert G == min(sms, 160, max(1, (2 * P.n_vals + P.n_meta) // (2 * b1 * b2)))
    vo, mo = orc.offsets(n, k, b1, b2, tmap)
    Pb = 2 * vo.astype(np.int64) + mo
    rec = plan[8: 8 + 4 * (G + 1)].reshape(G + 1, 4)
    starts = _tile_split_reference(Pb, G)
    assert list(rec[:, 0]) == starts
    tpr, tpd = k // b2, max(1, 16384 // (b1 * b2))
    for c in range(G):
        t0, t1 = starts[c], starts[c + 1]
        assert (rec[c, 1], rec[c, 2]) == (vo[t0], mo[t0]), c
        nw = min(31, t1 - t0)
        bits = sum(1 << i for i in range(nw) if tmap[t0 + i] == 1)
        word = int(rec[c, 3]) & 0xFFFFFFFFFFFFFFFF
        assert word & 0xFFFFFFFF == bits, c
        # stage starts of the first window: greedy by value bytes (a 2:4 tile
        # is one unit, a dense tile two), at most 2 tpd units and 2 tpd tiles
        # per stage, a new stage at every band start
        want, fill, cnt = 0, 4 * tpd, 2 * tpd
        for i in range(nw):
            sz = 1 if tmap[t0 + i] == 1 else 2
            if (t0 + i) % tpr == 0 or fill + sz > 2 * tpd or cnt == 2 * tpd:
                want |= 1 << i
                fill, cnt = 0, 0
            fill += sz
            cnt += 1
        assert word >> 32 == want, c
    Xd = X.to(dev())
    y_plan = hyb.spmv(P, Xd)
    saved = P.plan
    P.plan = None
    y_search = hyb.spmv(P, Xd)
    P.plan, P.plan_ctas = saved, G + 1  # a plan for another CTA count is ignored
    y_stale = hyb.spmv(P, Xd)
    assert torch.equal(y_plan, y_search) and torch.equal(y_plan, y_stale)
    y_ref, env = orc.spmv(n, k, b1, b2, tmap, orc.pack(inputs.bits(W), b1, b2, tmap),
                          inputs.bits(X))
    assert_within(y_plan.cpu().numpy().reshape(-1), y_ref.reshape(-1), env.reshape(-1),
                  what="plan")


def test_cuda_graph_capture_replay():
    """hyb_spmm_skinny launches nothing but kernels on the given stream, so it
    can be captured in a CUDA graph; replays give the eager result."""
    tmap = inputs.attn_map(1024)
    W, tmap, X, _ = case(4096, 4096, 128, 128, tmap, batch=2, name="attn_4096")
    P = hyb.pack(W.to(dev()), tmap, 128, 128)
    Xd = X.to(dev())
    ws = hyb.new_workspace(hyb.workspace_bytes(P, 2), dev())
    y_eager = hyb.spmm_skinny(P, Xd, ws=ws).clone()
    Y = torch.empty_like(y_eager)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        hyb.spmm_skinny(P, Xd, Y=Y, ws=ws)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        hyb.spmm_skinny(P, Xd, Y=Y, ws=ws)
    Y.zero_()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y, y_eager)
