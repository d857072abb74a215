"""CPU oracle for the tile-hybrid (dense | 2:4) weight format -- TEST INFRASTRUCTURE.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It wraps the plain C routines of
``hyb_oracle.c`` (fp64 products, loops that follow the definitions) with numpy
marshalling and shares no code with the CUDA library.

All bf16 data crosses as ``numpy.uint16`` arrays holding the raw bit patterns.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int

_libs = {}


def load(mutant: int = 0, path: str = None):
    """Load (building first if needed) the oracle library; ``mutant`` selects a
    variant with one planted mistake, used only by the pin-sensitivity tests."""
    key = (mutant, path)
    if key in _libs:
        return _libs[key]
    if path is None:
        path = _build.DEFAULT_OUT if mutant == 0 else os.path.join(
            _build.HERE, f"libhyb_oracle_mut{mutant}.so")
    _build.build(mutant=mutant, out=path)
    lib = ctypes.CDLL(path)
    lib.oracle_packed_sizes.argtypes = [_I64, _I64, _I, _I, _P, _P, _P]
    lib.oracle_packed_sizes.restype = _I
    lib.oracle_offsets.argtypes = [_I64, _I64, _I, _I, _P, _P, _P]
    lib.oracle_offsets.restype = _I
    lib.oracle_pack.argtypes = [_I64, _I64, _I, _I, _P, _I64, _P, _P, _P, _P, _P]
    lib.oracle_pack.restype = _I64
    lib.oracle_unpack.argtypes = [_I64, _I64, _I, _I, _P, _P, _P, _P, _P, _P]
    lib.oracle_unpack.restype = _I
    lib.oracle_matvec_f64.argtypes = [_I64, _I64, _P, _I64, _I, _P, _I64, _P,
                                      _I64, _P, _I64, _I, _P, _I64, _P]
    lib.oracle_matvec_f64.restype = _I
    lib.oracle_spmv_f64.argtypes = [_I64, _I64, _I, _I, _P, _P, _P, _P, _P, _I,
                                    _P, _I64, _P, _I64, _P, _I64, _I, _P, _I64, _P]
    lib.oracle_spmv_f64.restype = _I
    lib.oracle_rows_f64.argtypes = [_I64, _I64, _I, _I, _P, _I64, _P, _I, _P,
                                    _I64, _P, _I64, _P, _I64, _I, _P, _I64, _P, _P]
    lib.oracle_rows_f64.restype = _I
    lib.oracle_bf16_to_f64.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_to_f64.restype = ctypes.c_double
    lib.oracle_offsets_nm.argtypes = [_I64, _I64, _I, _I, _I, _I, _P, _P, _P]
    lib.oracle_offsets_nm.restype = _I
    lib.oracle_pack_nm.argtypes = [_I64, _I64, _I, _I, _I, _I, _P, _I64, _P, _P, _P, _P, _P]
    lib.oracle_pack_nm.restype = _I64
    lib.oracle_unpack_nm.argtypes = [_I64, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]
    lib.oracle_unpack_nm.restype = _I
    lib.oracle_spmv_nm_f64.argtypes = [_I64, _I64, _I, _I, _I, _I, _P, _P, _P, _P, _P, _I,
                                       _P, _I64, _P, _I64, _P, _I64, _I, _P, _I64, _P]
    lib.oracle_spmv_nm_f64.restype = _I
    _libs[key] = lib
    return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    pass


class Oracle:
    """numpy front end of one build of the C oracle."""

    def __init__(self, mutant: int = 0):
        self.lib = load(mutant)

    def packed_sizes(self, n, k, b1, b2, tile_map):
        tile_map = _c(tile_map, np.uint8)
        nv, nm = _I64(), _I64()
        rc = self.lib.oracle_packed_sizes(n, k, b1, b2, _ptr(tile_map),
                                          ctypes.byref(nv), ctypes.byref(nm))
        if rc != 0:
            raise OracleError("oracle_packed_sizes: bad argument")
        return nv.value, nm.value

    def offsets(self, n, k, b1, b2, tile_map):
        tile_map = _c(tile_map, np.uint8)
        T = tile_map.size
        vo = np.zeros(T + 1, np.int64)
        mo = np.zeros(T + 1, np.int64)
        if self.lib.oracle_offsets(n, k, b1, b2, _ptr(tile_map), _ptr(vo), _ptr(mo)) != 0:
            raise OracleError("oracle_offsets: bad argument")
        return vo, mo

    def pack(self, W, b1, b2, tile_map):
        """Returns dict(vals, meta, val_off, meta_off, nan_groups)."""
        W = _c(W, np.uint16)
        n, k = W.shape
        tile_map = _c(tile_map, np.uint8).reshape(-1)
        nv, nm = self.packed_sizes(n, k, b1, b2, tile_map)
        vals = np.zeros(nv, np.uint16)
        meta = np.zeros(max(nm, 1), np.uint8)
        vo = np.zeros(tile_map.size + 1, np.int64)
        mo = np.zeros(tile_map.size + 1, np.int64)
        rc = self.lib.oracle_pack(n, k, b1, b2, _ptr(W), k, _ptr(tile_map),
                                  _ptr(vals), _ptr(meta), _ptr(vo), _ptr(mo))
        if rc < 0:
            raise OracleError("oracle_pack: bad argument")
        return dict(vals=vals, meta=meta[:nm], val_off=vo, meta_off=mo,
                    nan_groups=int(rc))

    def unpack(self, n, k, b1, b2, tile_map, packed):
        tile_map = _c(tile_map, np.uint8).reshape(-1)
        W_hat = np.zeros((n, k), np.uint16)
        meta = packed["meta"] if packed["meta"].size else np.zeros(1, np.uint8)
        rc = self.lib.oracle_unpack(n, k, b1, b2, _ptr(tile_map),
                                    _ptr(_c(packed["vals"], np.uint16)),
                                    _ptr(_c(meta, np.uint8)),
                                    _ptr(_c(packed["val_off"], np.int64)),
                                    _ptr(_c(packed["meta_off"], np.int64)),
                                    _ptr(W_hat))
        if rc != 0:
            raise OracleError("oracle_unpack: bad argument")
        return W_hat

    def matvec(self, A, X, U=None, V=None):
        """fp64 Y[b][i] = (A x_b)_i (+ (U (V^T x_b))_i) and its envelope."""
        A = _c(A, np.uint16)
        X = np.atleast_2d(_c(X, np.uint16))
        n, k = A.shape
        batch = X.shape[0]
        rank = 0 if U is None else U.shape[1]
        U = _c(U, np.uint16)
        V = _c(V, np.uint16)
        Y = np.zeros((batch, n), np.float64)
        env = np.zeros((batch, n), np.float64)
        rc = self.lib.oracle_matvec_f64(n, k, _ptr(A), k, batch, _ptr(X), X.shape[1],
                                        _ptr(U), rank if rank else 1, _ptr(V),
                                        rank if rank else 1, rank, _ptr(Y), n, _ptr(env))
        if rc != 0:
            raise OracleError("oracle_matvec_f64: bad argument")
        return Y, env

    def spmv(self, n, k, b1, b2, tile_map, packed, X, U=None, V=None):
        tile_map = _c(tile_map, np.uint8).reshape(-1)
        X = np.atleast_2d(_c(X, np.uint16))
        batch = X.shape[0]
        rank = 0 if U is None else U.shape[1]
        U = _c(U, np.uint16)
        V = _c(V, np.uint16)
        meta = packed["meta"] if packed["meta"].size else np.zeros(1, np.uint8)
        Y = np.zeros((batch, n), np.float64)
        env = np.zeros((batch, n), np.float64)
        rc = self.lib.oracle_spmv_f64(n, k, b1, b2, _ptr(tile_map),
                                      _ptr(_c(packed["vals"], np.uint16)),
                                      _ptr(_c(meta, np.uint8)),
                                      _ptr(_c(packed["val_off"], np.int64)),
                                      _ptr(_c(packed["meta_off"], np.int64)),
                                      batch, _ptr(X), X.shape[1], _ptr(U),
                                      rank if rank else 1, _ptr(V), rank if rank else 1,
                                      rank, _ptr(Y), n, _ptr(env))
        if rc != 0:
            raise OracleError("oracle_spmv_f64: bad argument")
        return Y, env

    def rows(self, W, b1, b2, tile_map, X, rows, U=None, V=None):
        """fp64 hybrid product for selected output rows, from dense W + map."""
        W = _c(W, np.uint16)
        n, k = W.shape
        tile_map = _c(tile_map, np.uint8).reshape(-1)
        X = np.atleast_2d(_c(X, np.uint16))
        batch = X.shape[0]
        rows = _c(rows, np.int64)
        rank = 0 if U is None else U.shape[1]
        U = _c(U, np.uint16)
        V = _c(V, np.uint16)
        Y = np.zeros((batch, rows.size), np.float64)
        env = np.zeros((batch, rows.size), np.float64)
        rc = self.lib.oracle_rows_f64(n, k, b1, b2, _ptr(W), k, _ptr(tile_map), batch,
                                      _ptr(X), X.shape[1], _ptr(U), rank if rank else 1,
                                      _ptr(V), rank if rank else 1, rank, _ptr(rows),
                                      rows.size, _ptr(Y), _ptr(env))
        if rc != 0:
            raise OracleError("oracle_rows_f64: bad argument")
        return Y, env

    def bf16_to_f64(self, h):
        return self.lib.oracle_bf16_to_f64(int(h))

    # ---- general N:M tiles (nk kept of every m columns) ----

    def offsets_nm(self, n, k, b1, b2, nk, m, tile_map):
        tile_map = _c(tile_map, np.uint8).reshape(-1)
        vo = np.zeros(tile_map.size + 1, np.int64)
        mo = np.zeros(tile_map.size + 1, np.int64)
        if self.lib.oracle_offsets_nm(n, k, b1, b2, nk, m, _ptr(tile_map), _ptr(vo),
                                      _ptr(mo)) != 0:
            raise OracleError("oracle_offsets_nm: bad argument")
        return vo, mo

    def pack_nm(self, W, b1, b2, tile_map, nk, m):
        """Returns dict(vals, meta, val_off, meta_off, nan_groups)."""
        W = _c(W, np.uint16)
        n, k = W.shape
        tile_map = _c(tile_map, np.uint8).reshape(-1)
        vo, mo = self.offsets_nm(n, k, b1, b2, nk, m, tile_map)
        vals = np.zeros(int(vo[-1]), np.uint16)
        meta = np.zeros(max(int(mo[-1]), 1), np.uint8)
        rc = self.lib.oracle_pack_nm(n, k, b1, b2, nk, m, _ptr(W), k, _ptr(tile_map),
                                     _ptr(vals), _ptr(meta), _ptr(vo), _ptr(mo))
        if rc < 0:
            raise OracleError("oracle_pack_nm: bad argument")
        return dict(vals=vals, meta=meta[:int(mo[-1])], val_off=vo, meta_off=mo,
                    nan_groups=int(rc))

    def unpack_nm(self, n, k, b1, b2, nk, m, tile_map, packed):
        tile_map = _c(tile_map, np.uint8).reshape(-1)
        W_hat = np.zeros((n, k), np.uint16)
        meta = packed["meta"] if packed["meta"].size else np.zeros(1, np.uint8)
        rc = self.lib.oracle_unpack_nm(n, k, b1, b2, nk, m, _ptr(tile_map),
                                       _ptr(_c(packed["vals"], np.uint16)),
                                       _ptr(_c(meta, np.uint8)),
                                       _ptr(_c(packed["val_off"], np.int64)),
                                       _ptr(_c(packed["meta_off"], np.int64)),
                                       _ptr(W_hat))
        if rc != 0:
            raise OracleError("oracle_unpack_nm: bad argument")
        return W_hat

    def spmv_nm(self, n, k, b1, b2, nk, m, tile_map, packed, X, U=None, V=None):
        tile_map = _c(tile_map, np.uint8).reshape(-1)
        X = np.atleast_2d(_c(X, np.uint16))
        batch = X.shape[0]
        rank = 0 if U is None else U.shape[1]
        U = _c(U, np.uint16)
        V = _c(V, np.uint16)
        meta = packed["meta"] if packed["meta"].size else np.zeros(1, np.uint8)
        Y = np.zeros((batch, n), np.float64)
        env = np.zeros((batch, n), np.float64)
        rc = self.lib.oracle_spmv_nm_f64(n, k, b1, b2, nk, m, _ptr(tile_map),
                                         _ptr(_c(packed["vals"], np.uint16)),
                                         _ptr(_c(meta, np.uint8)),
                                         _ptr(_c(packed["val_off"], np.int64)),
                                         _ptr(_c(packed["meta_off"], np.int64)),
                                         batch, _ptr(X), X.shape[1], _ptr(U),
                                         rank if rank else 1, _ptr(V), rank if rank else 1,
                                         rank, _ptr(Y), n, _ptr(env))
        if rc != 0:
            raise OracleError("oracle_spmv_nm_f64: bad argument")
        return Y, env
