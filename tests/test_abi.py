"""The C ABI without a GPU: the library loads, exports every entry point
declared in include/hyb.h, and rejects bad arguments synchronously (these
checks run before any CUDA call, so they are safe on a machine with no GPU)."""
import ctypes
import os
import re

import numpy as np
import pytest

from sparse_weight_b200 import hyb

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "hyb.h")).read()
    return sorted(set(re.findall(r"HYB_API\s+[\w\s\*]*?\b(hyb_\w+)\s*\(", txt)))


@pytest.fixture(scope="module")
def L():
    from sparse_weight_b200 import build
    build.build()
    return hyb.lib()


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert len(names) >= 13
    for name in names:
        assert hasattr(L, name), name
    assert set(hyb.EXPORTS) == set(names)


def test_status_strings(L):
    for code in range(0, -8, -1):
        assert hyb.status_string(code) and "unknown" not in hyb.status_string(code)
    assert "unknown" in hyb.status_string(-99)


def test_selftest_argument_checks(L):
    """The failure-path self test validates its arguments before any launch."""
    f = L.hyb_selftest_wait_timeout
    assert f(None, 256, 10, None) == hyb.HYB_ERR_WORKSPACE
    assert f(ctypes.c_void_p(256), 255, 10, None) == hyb.HYB_ERR_WORKSPACE
    assert f(ctypes.c_void_p(256 + 16), 256, 10, None) == hyb.HYB_ERR_ALIGNMENT
    assert f(ctypes.c_void_p(256), 256, 0, None) == hyb.HYB_ERR_INVALID_ARG
    assert f(ctypes.c_void_p(256), 256, (1 << 20) + 1, None) == hyb.HYB_ERR_INVALID_ARG


def _sizes(n, k, b1, b2, m):
    m = np.ascontiguousarray(m, np.uint8)
    nv, nm = ctypes.c_int64(), ctypes.c_int64()
    rc = hyb.lib().hyb_packed_sizes(n, k, b1, b2, m.ctypes.data_as(ctypes.c_void_p),
                                    ctypes.byref(nv), ctypes.byref(nm))
    return rc, nv.value, nm.value


def test_packed_sizes_closed_form(L, orc):
    rng = np.random.default_rng(0)
    for (n, k, b1, b2) in [(256, 256, 64, 64), (4096, 4096, 128, 128), (1024, 4096, 128, 64),
                           (64, 96, 16, 32), (64, 128, 16, 8), (128, 96, 64, 24)]:
        T = (n // b1) * (k // b2)
        m = (rng.random(T) < 0.5).astype(np.uint8)
        rc, nv, nm = _sizes(n, k, b1, b2, m)
        assert rc == hyb.HYB_OK
        assert (nv, nm) == orc.packed_sizes(n, k, b1, b2, m)
        s = int(m.sum())
        assert nv == (T - s) * b1 * b2 + s * b1 * b2 // 2 and nm == s * b1 * b2 // 8


@pytest.mark.parametrize("shape", [(0, 64, 16, 16), (64, 64, 8, 8), (64, 64, 32, 4),
                                   (60, 64, 16, 16), (64, 60, 16, 16), (8, 16, 1, 16),
                                   (64, 60, 16, 12)])
def test_packed_sizes_rejects_bad_tiling(L, shape):
    n, k, b1, b2 = shape
    T = max(1, (n // max(b1, 1)) * (k // max(b2, 1)))
    rc, _, _ = _sizes(n, k, b1, b2, np.zeros(T, np.uint8))
    assert rc == hyb.HYB_ERR_INVALID_ARG


def test_packed_sizes_rejects_bad_map_byte(L):
    m = np.zeros(16, np.uint8)
    m[3] = 2
    rc, _, _ = _sizes(256, 256, 64, 64, m)
    assert rc == hyb.HYB_ERR_INVALID_ARG


def test_pack_argument_checks(L):
    P = ctypes.c_void_p
    good = P(0x10000)
    odd = P(0x10008)
    # null W
    assert L.hyb_pack(64, 64, 16, 16, None, 64, good, good, good, good, good, good, 256,
                      None) == hyb.HYB_ERR_INVALID_ARG
    # ldw < k
    assert L.hyb_pack(64, 64, 16, 16, good, 32, good, good, good, good, good, good, 256,
                      None) == hyb.HYB_ERR_INVALID_ARG
    # no workspace
    assert L.hyb_pack(64, 64, 16, 16, good, 64, good, good, good, good, good, None, 0,
                      None) == hyb.HYB_ERR_WORKSPACE
    # misaligned W
    assert L.hyb_pack(64, 64, 16, 16, odd, 64, good, good, good, good, good, good, 256,
                      None) == hyb.HYB_ERR_ALIGNMENT


def _matrix(**kw):
    d = dict(n=256, k=256, b1=64, b2=64, num_tiles=16, tile_map=0x10000, vals=0x20000,
             meta=0x30000, val_off=0x40000, meta_off=0x50000, n_vals=256 * 256,
             n_meta_bytes=0)
    d.update(kw)
    return hyb.HybMatrix(**d)


def test_spmv_argument_checks(L):
    P = ctypes.c_void_p
    X, Y, ws = P(0x60000), P(0x70000), P(0x80000)
    A = _matrix()
    call = lambda A, X=X, ldx=256, Y=Y, ldy=256, ydt=0, lr=None: L.hyb_spmv(
        ctypes.byref(A), X, ldx, Y, ldy, ydt, lr, ws, 1 << 20, None)
    assert L.hyb_spmv(None, X, 256, Y, 256, 0, None, ws, 1 << 20, None) == hyb.HYB_ERR_INVALID_ARG
    assert call(_matrix(num_tiles=15)) == hyb.HYB_ERR_INVALID_ARG
    assert call(_matrix(vals=None)) == hyb.HYB_ERR_INVALID_ARG
    assert call(_matrix(meta=None)) == hyb.HYB_ERR_INVALID_ARG
    assert call(_matrix(n_vals=5)) == hyb.HYB_ERR_INVALID_ARG
    assert call(_matrix(vals=0x20010)) == hyb.HYB_ERR_ALIGNMENT
    assert call(A, X=None) == hyb.HYB_ERR_INVALID_ARG
    assert call(A, ldx=100) == hyb.HYB_ERR_INVALID_ARG
    assert call(A, ldx=260) == hyb.HYB_ERR_ALIGNMENT
    assert call(A, X=P(0x60002)) == hyb.HYB_ERR_ALIGNMENT
    assert call(A, Y=P(0x70002)) == hyb.HYB_ERR_ALIGNMENT  # fp32 Y needs 4 bytes
    assert call(A, ydt=7) == hyb.HYB_ERR_INVALID_ARG
    lr = hyb.HybLowrank(12, 0x90000, 16, 0xA0000, 16)
    assert call(A, lr=ctypes.byref(lr)) == hyb.HYB_ERR_UNSUPPORTED
    lr = hyb.HybLowrank(16, None, 16, 0xA0000, 16)
    assert call(A, lr=ctypes.byref(lr)) == hyb.HYB_ERR_INVALID_ARG
    lr = hyb.HybLowrank(512, 0x90000, 512, 0xA0000, 512)
    assert call(A, lr=ctypes.byref(lr)) == hyb.HYB_ERR_INVALID_ARG
    # batch out of range
    assert L.hyb_spmm_skinny(ctypes.byref(A), 17, X, 256, Y, 256, 0, None, ws, 1 << 20,
                             None) == hyb.HYB_ERR_INVALID_ARG
    assert L.hyb_spmm_skinny(ctypes.byref(A), 0, X, 256, Y, 256, 0, None, ws, 1 << 20,
                             None) == hyb.HYB_ERR_INVALID_ARG


def test_launch_flags_checked(L):
    """The _ex entry points reject unknown launch-option bits before anything
    is queued (the valid bit, HYB_LAUNCH_OVERLAP_PREV, is exercised on the GPU)."""
    P = ctypes.c_void_p
    A = _matrix()
    X, Y, ws = P(0x60000), P(0x70000), P(0x80000)
    for flags in (2, 0x80000000, 3):
        assert L.hyb_spmm_skinny_ex(ctypes.byref(A), 1, X, 256, Y, 256, 0, None, flags, ws,
                                    1 << 20, None) == hyb.HYB_ERR_INVALID_ARG
        assert L.hyb_gemv_dense_ex(64, 64, 1, P(0x10000), 64, X, 64, Y, 64, 0, flags, ws,
                                   1 << 20, None) == hyb.HYB_ERR_INVALID_ARG
    # the flag does not bypass the other checks
    assert L.hyb_spmm_skinny_ex(ctypes.byref(A), 17, X, 256, Y, 256, 0, None,
                                hyb.LAUNCH_OVERLAP_PREV, ws, 1 << 20,
                                None) == hyb.HYB_ERR_INVALID_ARG
    assert L.hyb_gemv_dense_ex(64, 40, 1, P(0x10000), 40, X, 40, Y, 64, 0,
                               hyb.LAUNCH_OVERLAP_PREV, ws, 1 << 20,
                               None) == hyb.HYB_ERR_INVALID_ARG


def test_nm_sizes_and_argument_checks(L, orc):
    """hyb_packed_sizes_nm (host only) against the oracle's offsets, and the
    N:M entry points' synchronous argument checks."""
    rng = np.random.default_rng(5)
    for (nk, m) in [(1, 4), (2, 4), (3, 4), (2, 8), (4, 8), (6, 8), (4, 16), (8, 16)]:
        n, k, b1, b2 = 256, 512, 64, 64
        tmap = (rng.random((n // b1) * (k // b2)) < 0.5).astype(np.uint8)
        nv, nmb = hyb.packed_sizes_nm(n, k, b1, b2, nk, m, tmap)
        vo, mo = orc.offsets_nm(n, k, b1, b2, nk, m, tmap)
        assert (nv, nmb) == (int(vo[-1]), int(mo[-1])), (nk, m)
    # 2:4 through the N:M entry point is the 2:4 format
    assert hyb.packed_sizes_nm(n, k, b1, b2, 2, 4, tmap) == hyb.packed_sizes(n, k, b1, b2, tmap)
    P = ctypes.c_void_p
    tm = np.zeros(64, np.uint8)
    out = (ctypes.c_int64(), ctypes.c_int64())
    sizes = lambda nk, m: L.hyb_packed_sizes_nm(
        256, 512, 64, 64, nk, m, tm.ctypes.data_as(P), ctypes.byref(out[0]), ctypes.byref(out[1]))
    assert sizes(4, 8) == hyb.HYB_OK
    assert sizes(3, 6) == hyb.HYB_ERR_UNSUPPORTED
    assert sizes(0, 8) == hyb.HYB_ERR_INVALID_ARG
    assert sizes(8, 8) == hyb.HYB_ERR_INVALID_ARG
    W, X, Y, ws = P(0x10000), P(0x60000), P(0x70000), P(0x80000)
    assert L.hyb_pack_nm(256, 256, 64, 64, 4, 8, W, 256, P(0x20000), P(0x30000), P(0x40000),
                         P(0x50000), P(0x58000), None, 0, None) == hyb.HYB_ERR_WORKSPACE
    assert L.hyb_pack_nm(256, 256, 64, 64, 5, 6, W, 256, P(0x20000), P(0x30000), P(0x40000),
                         P(0x50000), P(0x58000), ws, 1 << 20, None) == hyb.HYB_ERR_UNSUPPORTED
    A = _matrix(n_vals=256 * 256 // 2, n_meta_bytes=256 * 256 // 8)
    call = lambda A, nk=4, m=8, batch=1, X=X: L.hyb_spmm_skinny_nm(
        ctypes.byref(A), nk, m, batch, X, 256, Y, 256, 0, ws, 1 << 20, None)
    assert call(A, batch=17) == hyb.HYB_ERR_INVALID_ARG
    assert call(A, nk=9) == hyb.HYB_ERR_INVALID_ARG
    assert call(A, m=6) == hyb.HYB_ERR_UNSUPPORTED
    assert call(A, X=None) == hyb.HYB_ERR_INVALID_ARG
    assert call(A, X=P(0x60008)) == hyb.HYB_ERR_ALIGNMENT
    assert call(_matrix(n_vals=5)) == hyb.HYB_ERR_INVALID_ARG
    assert L.hyb_spmm_skinny_nm(None, 4, 8, 1, X, 256, Y, 256, 0, ws, 1 << 20,
                                None) == hyb.HYB_ERR_INVALID_ARG
    assert L.hyb_spmm_skinny_nm(ctypes.byref(A), 4, 8, 1, X, 256, Y, 256, 0, None, 0,
                                None) == hyb.HYB_ERR_WORKSPACE


def test_dense_and_lowrank_argument_checks(L):
    P = ctypes.c_void_p
    W, X, Y, ws = P(0x10000), P(0x60000), P(0x70000), P(0x80000)
    assert L.hyb_gemv_dense(64, 40, 1, W, 40, X, 40, Y, 64, 0, ws, 1 << 20,
                            None) == hyb.HYB_ERR_INVALID_ARG  # k % 16
    assert L.hyb_gemv_dense(64, 64, 1, P(0x10008), 64, X, 64, Y, 64, 0, ws, 1 << 20,
                            None) == hyb.HYB_ERR_ALIGNMENT  # W not 16-byte aligned
    assert L.hyb_gemv_dense(64, 64, 1, W, 68, X, 64, Y, 64, 0, ws, 1 << 20,
                            None) == hyb.HYB_ERR_ALIGNMENT  # rows not 16-byte aligned
    assert L.hyb_gemv_dense(60, 48, 1, W, 52, X, 48, Y, 64, 0, ws, 1 << 20,
                            None) == hyb.HYB_ERR_ALIGNMENT
    lr = hyb.HybLowrank(0, P(0x90000), 8, P(0xA0000), 8)
    assert L.hyb_lowrank_add(64, 64, 1, ctypes.byref(lr), X, 64, Y, 64, ws, 1 << 20,
                             None) == hyb.HYB_ERR_INVALID_ARG
    assert L.hyb_workspace_bytes(None, 1, 0) == 0
    A = _matrix(b2=4)
    assert L.hyb_workspace_bytes(ctypes.byref(A), 1, 0) == 0
    assert L.hyb_workspace_init(None, 0, None) == hyb.HYB_ERR_WORKSPACE
    assert L.hyb_check_status(None, None, None) == hyb.HYB_ERR_WORKSPACE
