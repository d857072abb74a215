"""Pins of the CPU oracle against what the pages and plain mathematics fix.

Each ``pin_*`` function takes an ``oracle.Oracle`` and raises AssertionError on
a mismatch.  They are run on the real oracle by ``test_oracle_pins.py`` and on
variants with one planted mistake by ``test_oracle_mutants.py`` (to show that
every planted mistake is caught).  None of them re-types the oracle's code:
they use a hand-worked fixture, brute-force enumeration, exact integer
arithmetic and closed forms.

Definitions pinned (see the oracle header for the full reading):
  * PATCH: Learnable Tile-level Hybrid Sparsity for LLMs, §2 Methodology --
    b1 x b2 tiles, each dense or 2:4; §2 pattern selection -- 6 patterns per
    group; §3 Contributions -- sparsity anywhere in 0..50 %.
  * SparseDecoding, authors' abstract -- bitmask-indexed, fixed-stride N:M.
  * 3BASiL, §1 Problem / §2A -- W ~ S + L with L = U V^T of rank r; magnitude
    projection for the sparse block.
"""
import itertools
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

PATTERNS = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]  # C(4,2), lexicographic


def f2bits(vals) -> np.ndarray:
    """bf16 bit patterns of values that bf16 represents exactly."""
    f = np.asarray(vals, dtype=np.float32)
    u = f.view(np.uint32)
    assert np.all(u & 0xFFFF == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


def round_bits(vals) -> np.ndarray:
    """bf16 bit patterns of arbitrary values, rounded to nearest even."""
    t = torch.tensor(np.asarray(vals, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bits2f(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def read_golden(name):
    d = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            key, *rest = line.split()
            d[key] = rest
    return d


def _ints_exact(W_hat_bits, X_bits, U_bits=None, V_bits=None):
    """Exact product for integer-valued bf16 data (Python ints, no rounding)."""
    A = bits2f(W_hat_bits)
    X = bits2f(X_bits)
    assert np.all(A == np.round(A)) and np.all(X == np.round(X))
    Ai = A.astype(np.int64)
    Xi = X.astype(np.int64)
    Y = Xi @ Ai.T  # int64, exact at these sizes
    E = np.abs(Xi) @ np.abs(Ai).T
    if U_bits is not None:
        Ui = bits2f(U_bits).astype(np.int64)
        Vi = bits2f(V_bits).astype(np.int64)
        T = Xi @ Vi              # batch x r
        Y = Y + T @ Ui.T
        E = E + (np.abs(Xi) @ np.abs(Vi)) @ np.abs(Ui).T
    return Y, E


def brute_force_mask(W_bits, tile_map, b1, b2):
    """Masked dense matrix by enumerating the six 2:4 patterns of every group
    and keeping the one with the largest sum of |w| keys; among equal sums the
    lexicographically first pattern wins (that is: ties go to lower columns)."""
    n, k = W_bits.shape
    out = np.zeros_like(W_bits)
    tpr = k // b2
    key = (W_bits & 0x7FFF).astype(np.int64)
    for i in range(n):
        for c0 in range(0, k, 4):
            t = (i // b1) * tpr + c0 // b2
            if tile_map[t] == 0:
                out[i, c0:c0 + 4] = W_bits[i, c0:c0 + 4]
                continue
            best, best_s = None, -1
            for p in PATTERNS:
                s = key[i, c0 + p[0]] + key[i, c0 + p[1]]
                if s > best_s:
                    best, best_s = p, s
            for j in best:
                out[i, c0 + j] = W_bits[i, c0 + j]
    return out


def _tie_heavy_ints(rng, shape, lo=-3, hi=3):
    v = rng.integers(lo, hi + 1, size=shape).astype(np.float32)
    # sprinkle negative zeros among the zeros
    z = (v == 0) & (rng.random(shape) < 0.5)
    v[z] = -0.0
    return f2bits(v)


# ---------------------------------------------------------------------------

def pin_golden(o):
    """Hand-worked 4x16 example (tests/golden/pack_4x16.txt)."""
    g = read_golden("pack_4x16.txt")
    n, k, b1, b2 = (int(g[s][0]) for s in ("n", "k", "b1", "b2"))
    tmap = np.array([int(v) for v in g["tile_map"]], np.uint8)
    W = np.stack([f2bits([float(v) for v in g[f"W{i}"]]) for i in range(n)])
    p = o.pack(W, b1, b2, tmap)
    assert p["val_off"].tolist() == [int(v) for v in g["val_off"]], p["val_off"]
    assert p["meta_off"].tolist() == [int(v) for v in g["meta_off"]], p["meta_off"]
    assert p["vals"].tolist() == f2bits([float(v) for v in g["vals"]]).tolist(), p["vals"]
    assert p["meta"].tolist() == [int(v, 16) for v in g["meta"]], p["meta"]
    X = f2bits([[float(v) for v in g["x"]]])
    Y, _ = o.spmv(n, k, b1, b2, tmap, p, X)
    assert Y[0].tolist() == [float(v) for v in g["y"]], Y
    Yd, _ = o.matvec(W, X)
    assert Yd[0].tolist() == [float(v) for v in g["y_dense"]], Yd
    U = f2bits([[float(v)] for v in g["U"]])
    V = f2bits([[float(v)] for v in g["V"]])
    Yl, _ = o.spmv(n, k, b1, b2, tmap, p, X, U, V)
    assert Yl[0].tolist() == [float(v) for v in g["y_lowrank"]], Yl


def pin_bruteforce(o):
    """8x8 and 8x16 inputs with many ties: every tile map of up to 4 tiles,
    selection checked against pattern enumeration, products against exact
    integer arithmetic."""
    rng = np.random.default_rng(1234)
    for (n, k, b1, b2) in [(8, 8, 2, 8), (8, 8, 4, 8), (8, 16, 4, 8), (4, 16, 4, 8)]:
        T = (n // b1) * (k // b2)
        for trial in range(3):
            W = _tie_heavy_ints(rng, (n, k))
            X = _tie_heavy_ints(rng, (2, k))
            for bitsmap in itertools.product([0, 1], repeat=T):
                tmap = np.array(bitsmap, np.uint8)
                p = o.pack(W, b1, b2, tmap)
                W_hat = o.unpack(n, k, b1, b2, tmap, p)
                expect = brute_force_mask(W, tmap, b1, b2)
                assert np.array_equal(W_hat, expect), (n, k, b1, b2, bitsmap)
                Y, E = o.spmv(n, k, b1, b2, tmap, p, X)
                Yi, Ei = _ints_exact(expect, X)
                assert np.array_equal(Y, Yi.astype(np.float64)), (bitsmap, Y, Yi)
                assert np.array_equal(E, Ei.astype(np.float64))


def pin_invariants(o):
    """Format invariants on random normal weights: two kept per group, offsets
    in closed form, mask sparsity = 0.5 x the 2:4-tile fraction, total bytes."""
    rng = np.random.default_rng(7)
    for (n, k, b1, b2) in [(64, 128, 16, 32), (128, 64, 32, 16), (96, 96, 32, 32)]:
        T = (n // b1) * (k // b2)
        W = round_bits(rng.standard_normal((n, k)) * 0.02)
        for frac in (0.0, 0.25, 0.5, 1.0):
            tmap = np.zeros(T, np.uint8)
            tmap[rng.permutation(T)[: int(round(frac * T))]] = 1
            p = o.pack(W, b1, b2, tmap)
            s = int(tmap.sum())
            te = b1 * b2
            # closed-form offsets
            vo = np.concatenate([[0], np.cumsum(np.where(tmap == 1, te // 2, te))])
            mo = np.concatenate([[0], np.cumsum(np.where(tmap == 1, te // 8, 0))])
            assert np.array_equal(p["val_off"], vo) and np.array_equal(p["meta_off"], mo)
            # total bytes: (T - s) dense tiles of 2 B/weight, s tiles of 1.125 B/weight
            total = 2 * p["vals"].size + p["meta"].size
            assert total * 8 == (T - s) * 16 * te + s * 9 * te
            # every nibble has exactly two bits set
            nib = np.concatenate([p["meta"] & 0xF, p["meta"] >> 4])
            assert np.all(np.isin(nib, [3, 5, 6, 9, 10, 12])), np.unique(nib)
            # mask sparsity: dropped positions / all positions = 0.5 * s / T
            W_hat = o.unpack(n, k, b1, b2, tmap, p)
            tpr = k // b2
            # dropped positions, counted from the decoded masks of the 2:4 tiles
            dropped = 0
            for t in np.nonzero(tmap)[0]:
                m = p["meta"][p["meta_off"][t]:p["meta_off"][t + 1]]
                for byte in m:
                    dropped += 4 - bin(int(byte) & 0xF).count("1")
                    dropped += 4 - bin(int(byte) >> 4).count("1")
            assert dropped * T * 2 == n * k * s
            # the value block of each tile holds W at the kept positions, in order
            for t in range(T):
                r0, c0 = (t // tpr) * b1, (t % tpr) * b2
                blk_hat = W_hat[r0:r0 + b1, c0:c0 + b2]
                v = p["vals"][p["val_off"][t]:p["val_off"][t + 1]]
                if tmap[t] == 0:
                    assert np.array_equal(v, W[r0:r0 + b1, c0:c0 + b2].reshape(-1))
                else:
                    assert v.size * 2 == b1 * b2


def pin_all_dense(o):
    """An all-dense tile map reproduces the plain dense product exactly."""
    rng = np.random.default_rng(11)
    n, k, b1, b2 = 32, 64, 8, 16
    W = _tie_heavy_ints(rng, (n, k), -20, 20)
    X = _tie_heavy_ints(rng, (3, k), -5, 5)
    tmap = np.zeros((n // b1) * (k // b2), np.uint8)
    p = o.pack(W, b1, b2, tmap)
    assert np.array_equal(o.unpack(n, k, b1, b2, tmap, p), W)
    Y, _ = o.spmv(n, k, b1, b2, tmap, p, X)
    Yi, _ = _ints_exact(W, X)
    assert np.array_equal(Y, Yi.astype(np.float64))
    # and on real-valued data against numpy's fp64 product (different order)
    Wf = round_bits(rng.standard_normal((n, k)) * 0.02)
    Xf = round_bits(rng.standard_normal((2, k)))
    p = o.pack(Wf, b1, b2, tmap)
    Y, _ = o.spmv(n, k, b1, b2, tmap, p, Xf)
    ref = bits2f(Xf) @ bits2f(Wf).T
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)


def pin_all_sparse(o):
    """An all-2:4 tile map equals uniform 2:4 magnitude pruning, written here
    as a stable sort of each group by (-|w|, column)."""
    rng = np.random.default_rng(5)
    n, k, b1, b2 = 64, 128, 16, 64
    for data in range(2):
        if data == 0:
            W = round_bits(rng.standard_normal((n, k)))
        else:
            W = _tie_heavy_ints(rng, (n, k), -2, 2)
        tmap = np.ones((n // b1) * (k // b2), np.uint8)
        p = o.pack(W, b1, b2, tmap)
        W_hat = o.unpack(n, k, b1, b2, tmap, p)
        key = (W & 0x7FFF).astype(np.int64).reshape(n, k // 4, 4)
        order = np.argsort(-key, axis=2, kind="stable")[:, :, :2]
        keep = np.zeros((n, k // 4, 4), bool)
        np.put_along_axis(keep, order, True, axis=2)
        expect = np.where(keep.reshape(n, k), W, 0).astype(np.uint16)
        assert np.array_equal(W_hat, expect)


def pin_lowrank(o):
    """S x + U (V^T x) equals (S + U V^T) x exactly on integer data; U = 0
    leaves S x unchanged."""
    rng = np.random.default_rng(3)
    n, k, b1, b2, r = 16, 32, 8, 16, 3
    W = _tie_heavy_ints(rng, (n, k), -6, 6)
    X = _tie_heavy_ints(rng, (2, k), -3, 3)
    U = _tie_heavy_ints(rng, (n, r), -3, 3)
    V = _tie_heavy_ints(rng, (k, r), -3, 3)
    tmap = np.array([1, 0, 0, 1, 1, 1, 0, 1][: (n // b1) * (k // b2)], np.uint8)
    p = o.pack(W, b1, b2, tmap)
    W_hat = brute_force_mask(W, tmap, b1, b2)
    Y, E = o.spmv(n, k, b1, b2, tmap, p, X, U, V)
    S = bits2f(W_hat).astype(np.int64)
    L = bits2f(U).astype(np.int64) @ bits2f(V).astype(np.int64).T
    Xi = bits2f(X).astype(np.int64)
    assert np.array_equal(Y, (Xi @ (S + L).T).astype(np.float64))
    _, Ei = _ints_exact(W_hat, X, U, V)
    assert np.array_equal(E, Ei.astype(np.float64))
    Y0, _ = o.spmv(n, k, b1, b2, tmap, p, X, np.zeros_like(U), V)
    Ys, _ = o.spmv(n, k, b1, b2, tmap, p, X)
    assert np.array_equal(Y0, Ys)


def pin_rows(o):
    """The sampled-row product equals exact integer arithmetic on the
    brute-force masked matrix, with and without the low-rank term."""
    rng = np.random.default_rng(9)
    n, k, b1, b2, r = 32, 48, 8, 16, 2
    W = _tie_heavy_ints(rng, (n, k), -8, 8)
    X = _tie_heavy_ints(rng, (3, k), -4, 4)
    U = _tie_heavy_ints(rng, (n, r), -2, 2)
    V = _tie_heavy_ints(rng, (k, r), -2, 2)
    T = (n // b1) * (k // b2)
    tmap = (rng.random(T) < 0.5).astype(np.uint8)
    rows = np.array([0, 5, 31, 17, 8], np.int64)
    W_hat = brute_force_mask(W, tmap, b1, b2)
    for lr in (False, True):
        Yi, Ei = _ints_exact(W_hat, X, U if lr else None, V if lr else None)
        Y, E = o.rows(W, b1, b2, tmap, X, rows, U if lr else None, V if lr else None)
        assert np.array_equal(Y, Yi[:, rows].astype(np.float64))
        assert np.array_equal(E, Ei[:, rows].astype(np.float64))


def pin_special_values(o):
    """Magnitude order on special bf16 values: +/-inf outrank every finite
    value, -0 ties +0 (lower column wins), subnormals order by magnitude, and a
    NaN is reported as a data error while the pack still completes."""
    inf, ninf = np.uint16(0x7F80), np.uint16(0xFF80)
    sub1, sub2 = np.uint16(0x0001), np.uint16(0x8002)  # smallest subnormals
    rows = [
        [f2bits([1.0])[0], ninf, f2bits([3.0])[0], f2bits([-2.0])[0]],  # keep 1 (-inf), 2 (3)
        [np.uint16(0x8000), np.uint16(0x0000), np.uint16(0x8000), np.uint16(0)],  # keep 0,1
        [sub1, np.uint16(0), sub2, np.uint16(0x8001)],  # keep 2 (|2|), then 0 (tie with 3)
        [inf, f2bits([-2.0 ** 100])[0], ninf, f2bits([5.0])[0]],  # keep 0,2
    ]
    W = np.array([[*r, *r] for r in rows], np.uint16)  # 4 x 8, one 4x8 tile
    tmap = np.ones(1, np.uint8)
    p = o.pack(W, 4, 8, tmap)
    assert p["nan_groups"] == 0
    nib = [int(p["meta"][i]) & 0xF for i in range(4)]
    assert nib == [0b0110, 0b0011, 0b0101, 0b0101], nib
    assert p["vals"][0:2].tolist() == [ninf, f2bits([3.0])[0]]
    assert p["vals"][4:6].tolist() == [0x8000, 0x0000]  # row 1 starts at b2/2
    Wn = W.copy()
    Wn[0, 0] = 0x7FC0  # quiet NaN
    pn = o.pack(Wn, 4, 8, tmap)
    assert pn["nan_groups"] == 1
    assert int(pn["meta"][0]) & 0xF == 0b0011  # NaN key outranks -inf


# ---------------------------------------------------------------------------
# general N:M tiles (PATCH, "Future direction": other N:M patterns such as
# 4:8; SparseDecoding's N:M kernel with a bitmask and a fixed stride)

NM_CASES = [(1, 4), (2, 4), (3, 4), (2, 8), (4, 8), (6, 8)]


def brute_force_mask_nm(W_bits, tile_map, b1, b2, nk, m):
    """Masked dense matrix by enumerating every choice of nk columns out of m
    in each group of a sparse tile and keeping the one with the largest sum of
    |w| keys; among equal sums the lexicographically first choice wins."""
    n, k = W_bits.shape
    out = np.zeros_like(W_bits)
    tpr = k // b2
    key = (W_bits & 0x7FFF).astype(np.int64)
    choices = list(itertools.combinations(range(m), nk))
    for i in range(n):
        for c0 in range(0, k, m):
            t = (i // b1) * tpr + c0 // b2
            if tile_map[t] == 0:
                out[i, c0:c0 + m] = W_bits[i, c0:c0 + m]
                continue
            best, best_s = None, -1
            for ch in choices:
                s = sum(int(key[i, c0 + j]) for j in ch)
                if s > best_s:
                    best, best_s = ch, s
            for j in best:
                out[i, c0 + j] = W_bits[i, c0 + j]
    return out


def mask_bits(meta_row):
    """The bit stream of one tile row's mask bytes, bit c = column c."""
    return [(int(meta_row[c // 8]) >> (c % 8)) & 1 for c in range(8 * len(meta_row))]


def pin_nm_golden(o):
    """Hand-worked 2x32 example with a 4:8 tile and a dense tile
    (tests/golden/pack_nm_2x32_4of8.txt)."""
    g = read_golden("pack_nm_2x32_4of8.txt")
    n, k, b1, b2, nk, m = (int(g[s][0]) for s in ("n", "k", "b1", "b2", "nk", "m"))
    tmap = np.array([int(v) for v in g["tile_map"]], np.uint8)
    W = np.stack([f2bits([float(v) for v in g[f"W{i}"]]) for i in range(n)])
    p = o.pack_nm(W, b1, b2, tmap, nk, m)
    assert p["val_off"].tolist() == [int(v) for v in g["val_off"]], p["val_off"]
    assert p["meta_off"].tolist() == [int(v) for v in g["meta_off"]], p["meta_off"]
    assert p["vals"].tolist() == f2bits([float(v) for v in g["vals"]]).tolist(), p["vals"]
    assert p["meta"].tolist() == [int(v, 16) for v in g["meta"]], p["meta"]
    X = f2bits([[float(v) for v in g["x"]]])
    Y, _ = o.spmv_nm(n, k, b1, b2, nk, m, tmap, p, X)
    assert Y[0].tolist() == [float(v) for v in g["y"]], Y
    Yd, _ = o.spmv_nm(n, k, b1, b2, nk, m, np.zeros_like(tmap),
                      o.pack_nm(W, b1, b2, np.zeros_like(tmap), nk, m), X)
    assert Yd[0].tolist() == [float(v) for v in g["y_dense"]], Yd


def pin_nm_is_2of4(o):
    """With N = 2, M = 4 the N:M routines give the 2:4 format bit for bit
    (values, masks, offsets), on tie-heavy integers and every map of 4 tiles."""
    rng = np.random.default_rng(99)
    n, k, b1, b2 = 8, 32, 4, 16
    for trial in range(3):
        W = _tie_heavy_ints(rng, (n, k))
        for bitsmap in itertools.product([0, 1], repeat=4):
            tmap = np.array(bitsmap, np.uint8)
            a = o.pack(W, b1, b2, tmap)
            b = o.pack_nm(W, b1, b2, tmap, 2, 4)
            for key in ("vals", "meta", "val_off", "meta_off"):
                assert np.array_equal(a[key], b[key]), (key, bitsmap)


def pin_nm_bruteforce(o):
    """Every (N, M) of NM_CASES on tie-heavy integer inputs and every map of up
    to 4 tiles: selection against enumeration of the C(M, N) choices, products
    against exact integer arithmetic."""
    rng = np.random.default_rng(4321)
    for (nk, m) in NM_CASES:
        for (n, k, b1, b2) in [(4, 16, 2, 8), (4, 32, 4, 16)]:
            if b2 % m:
                continue
            T = (n // b1) * (k // b2)
            W = _tie_heavy_ints(rng, (n, k))
            X = _tie_heavy_ints(rng, (2, k))
            for bitsmap in itertools.product([0, 1], repeat=T):
                tmap = np.array(bitsmap, np.uint8)
                p = o.pack_nm(W, b1, b2, tmap, nk, m)
                W_hat = o.unpack_nm(n, k, b1, b2, nk, m, tmap, p)
                expect = brute_force_mask_nm(W, tmap, b1, b2, nk, m)
                assert np.array_equal(W_hat, expect), (nk, m, n, k, bitsmap)
                Y, E = o.spmv_nm(n, k, b1, b2, nk, m, tmap, p, X)
                Yi, Ei = _ints_exact(expect, X)
                assert np.array_equal(Y, Yi.astype(np.float64)), (nk, m, bitsmap)
                assert np.array_equal(E, Ei.astype(np.float64))


def pin_nm_invariants(o):
    """Format invariants on random normal weights: nk mask bits per group of m,
    offsets and total bytes in closed form, kept values in ascending column
    order (read back through the mask), all-sparse selection equal to a stable
    sort of the magnitudes."""
    rng = np.random.default_rng(11)
    for (nk, m) in [(4, 8), (2, 8), (8, 16)]:
        n, k, b1, b2 = 32, 64, 8, 32
        T = (n // b1) * (k // b2)
        W = round_bits(rng.normal(0, 1, (n, k)))
        tmap = (rng.random(T) < 0.5).astype(np.uint8)
        p = o.pack_nm(W, b1, b2, tmap, nk, m)
        s = int(tmap.sum())
        assert p["val_off"][-1] == (T - s) * b1 * b2 + s * b1 * b2 * nk // m
        assert p["meta_off"][-1] == s * b1 * b2 // 8
        for t in range(T):
            size_v = p["val_off"][t + 1] - p["val_off"][t]
            size_m = p["meta_off"][t + 1] - p["meta_off"][t]
            assert size_v == (b1 * b2 * nk // m if tmap[t] else b1 * b2)
            assert size_m == (b1 * b2 // 8 if tmap[t] else 0)
            if not tmap[t]:
                continue
            tr, tc = divmod(t, k // b2)
            for i in range(b1):
                mrow = p["meta"][p["meta_off"][t] + i * (b2 // 8):
                                 p["meta_off"][t] + (i + 1) * (b2 // 8)]
                bits = mask_bits(mrow)
                vrow = p["vals"][p["val_off"][t] + i * (b2 * nk // m):
                                 p["val_off"][t] + (i + 1) * (b2 * nk // m)]
                w = W[tr * b1 + i, tc * b2:(tc + 1) * b2]
                kept = [c for c in range(b2) if bits[c]]
                for g in range(b2 // m):
                    assert sum(bits[g * m:(g + 1) * m]) == nk
                assert vrow.tolist() == [int(w[c]) for c in kept]
        # all-sparse: a stable sort by descending magnitude picks the same columns
        ones = np.ones(T, np.uint8)
        W_hat = o.unpack_nm(n, k, b1, b2, nk, m, ones, o.pack_nm(W, b1, b2, ones, nk, m))
        mag = np.abs(bits2f(W)).reshape(n, k // m, m)
        order = np.argsort(-mag, axis=2, kind="stable")[:, :, :nk]
        keep = np.zeros_like(mag, dtype=bool)
        np.put_along_axis(keep, order, True, axis=2)
        assert np.array_equal(W_hat, np.where(keep.reshape(n, k), W, 0).astype(np.uint16))


ALL_PINS = [pin_golden, pin_bruteforce, pin_invariants, pin_all_dense,
            pin_all_sparse, pin_lowrank, pin_rows, pin_special_values,
            pin_nm_golden, pin_nm_is_2of4, pin_nm_bruteforce, pin_nm_invariants]
