"""Thin Python binding of libhyb (include/hyb.h): argument marshalling only.

Every step of the product runs in the CUDA library; PyTorch provides device
memory and the current stream.  Function names follow the C ABI without the
``hyb_`` prefix.  bf16 tensors cross as their raw 16-bit patterns.

If ``libhyb.so`` is missing the first call raises; there is no fallback.
"""
import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhyb.so")

HYB_OK = 0
HYB_ERR_INVALID_ARG = -1
HYB_ERR_UNSUPPORTED = -2
HYB_ERR_ALIGNMENT = -3
HYB_ERR_WORKSPACE = -4
HYB_ERR_CUDA = -5
HYB_ERR_DEVICE_CHECK = -6
HYB_ERR_TIMEOUT = -7

HYB_F32 = 0
HYB_BF16 = 1
LAUNCH_OVERLAP_PREV = 1  # HYB_LAUNCH_OVERLAP_PREV

STATUS_NAN = 1
STATUS_BAD_MAP = 2
STATUS_TIMEOUT = 4

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int
_SZ = ctypes.c_size_t


class HybMatrix(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int64), ("k", ctypes.c_int64),
                ("b1", ctypes.c_int32), ("b2", ctypes.c_int32),
                ("num_tiles", ctypes.c_int64),
                ("tile_map", _P), ("vals", _P), ("meta", _P),
                ("val_off", _P), ("meta_off", _P),
                ("n_vals", ctypes.c_int64), ("n_meta_bytes", ctypes.c_int64),
                ("plan", _P), ("plan_ctas", ctypes.c_int32)]


class HybLowrank(ctypes.Structure):
    _fields_ = [("rank", ctypes.c_int32), ("U", _P), ("ldu", ctypes.c_int64),
                ("V", _P), ("ldv", ctypes.c_int64)]


class HybError(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} ({status})")


_lib = None

EXPORTS = ["hyb_packed_sizes", "hyb_pack_workspace_bytes", "hyb_pack",
           "hyb_workspace_bytes", "hyb_workspace_init", "hyb_spmv",
           "hyb_spmm_skinny", "hyb_lowrank_workspace_bytes", "hyb_lowrank_add",
           "hyb_dense_workspace_bytes", "hyb_gemv_dense", "hyb_check_status",
           "hyb_status_string", "hyb_spmv_noalloc", "hyb_spmv_noalloc_max_scratch_bytes",
           "hyb_spmv_noalloc_check_status", "hyb_gate_up_workspace_bytes",
           "hyb_spmm_skinny_gate_up", "hyb_prefill_workspace_bytes", "hyb_spmm_prefill",
           "hyb_prefill_block_shape", "hyb_spmm_prefill_blocked", "hyb_shard_bands",
           "hyb_plan_entries", "hyb_make_plan", "hyb_selftest_wait_timeout",
           "hyb_spmm_skinny_ex", "hyb_gemv_dense_ex", "hyb_packed_sizes_nm",
           "hyb_pack_nm", "hyb_spmm_skinny_nm"]


def lib():
    """Load libhyb.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libhyb.so not built ({LIB_PATH}); run "
                           "`python -m sparse_weight_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    L.hyb_packed_sizes.argtypes = [_I64, _I64, _I, _I, _P, _P, _P]
    L.hyb_packed_sizes.restype = _I
    L.hyb_pack_workspace_bytes.argtypes = []
    L.hyb_pack_workspace_bytes.restype = _SZ
    L.hyb_pack.argtypes = [_I64, _I64, _I, _I, _P, _I64, _P, _P, _P, _P, _P, _P, _SZ, _P]
    L.hyb_pack.restype = _I
    L.hyb_workspace_bytes.argtypes = [ctypes.POINTER(HybMatrix), _I, _I]
    L.hyb_workspace_bytes.restype = _SZ
    L.hyb_workspace_init.argtypes = [_P, _SZ, _P]
    L.hyb_workspace_init.restype = _I
    L.hyb_spmv.argtypes = [ctypes.POINTER(HybMatrix), _P, _I64, _P, _I64, _I,
                           ctypes.POINTER(HybLowrank), _P, _SZ, _P]
    L.hyb_spmv.restype = _I
    L.hyb_spmm_skinny.argtypes = [ctypes.POINTER(HybMatrix), _I, _P, _I64, _P, _I64, _I,
                                  ctypes.POINTER(HybLowrank), _P, _SZ, _P]
    L.hyb_spmm_skinny.restype = _I
    L.hyb_spmm_skinny_ex.argtypes = [ctypes.POINTER(HybMatrix), _I, _P, _I64, _P, _I64, _I,
                                     ctypes.POINTER(HybLowrank), ctypes.c_uint32, _P, _SZ, _P]
    L.hyb_spmm_skinny_ex.restype = _I
    L.hyb_gate_up_workspace_bytes.argtypes = [ctypes.POINTER(HybMatrix), ctypes.POINTER(HybMatrix),
                                              _I, _I]
    L.hyb_gate_up_workspace_bytes.restype = _SZ
    L.hyb_spmm_skinny_gate_up.argtypes = [ctypes.POINTER(HybMatrix), ctypes.POINTER(HybMatrix), _I,
                                          _P, _I64, _P, _I64, _P, _I64, _I,
                                          ctypes.POINTER(HybLowrank), _P, _I64, ctypes.c_uint32,
                                          _P, _SZ, _P]
    L.hyb_spmm_skinny_gate_up.restype = _I
    L.hyb_shard_bands.argtypes = [_I64, _I64, _I, _I, _P, _I, _I, ctypes.POINTER(ctypes.c_int64),
                                  ctypes.POINTER(ctypes.c_int64)]
    L.hyb_shard_bands.restype = _I
    L.hyb_prefill_workspace_bytes.argtypes = []
    L.hyb_prefill_workspace_bytes.restype = _SZ
    L.hyb_spmm_prefill.argtypes = [ctypes.POINTER(HybMatrix), _I64, _P, _I64, _P, _I64, _P, _SZ,
                                   _P]
    L.hyb_spmm_prefill.restype = _I
    L.hyb_prefill_block_shape.argtypes = [_I64, _I64, ctypes.POINTER(_I), ctypes.POINTER(_I)]
    L.hyb_prefill_block_shape.restype = _I
    L.hyb_spmm_prefill_blocked.argtypes = [ctypes.POINTER(HybMatrix), _I64, _P, _I64, _P, _I64,
                                           _I, _I, _P, _SZ, _P]
    L.hyb_spmm_prefill_blocked.restype = _I
    L.hyb_lowrank_workspace_bytes.argtypes = [_I64, _I, _I]
    L.hyb_lowrank_workspace_bytes.restype = _SZ
    L.hyb_lowrank_add.argtypes = [_I64, _I64, _I, ctypes.POINTER(HybLowrank), _P, _I64,
                                  _P, _I64, _P, _SZ, _P]
    L.hyb_lowrank_add.restype = _I
    L.hyb_dense_workspace_bytes.argtypes = [_I64, _I64, _I]
    L.hyb_dense_workspace_bytes.restype = _SZ
    L.hyb_gemv_dense.argtypes = [_I64, _I64, _I, _P, _I64, _P, _I64, _P, _I64, _I, _P,
                                 _SZ, _P]
    L.hyb_gemv_dense.restype = _I
    L.hyb_gemv_dense_ex.argtypes = [_I64, _I64, _I, _P, _I64, _P, _I64, _P, _I64, _I,
                                    ctypes.c_uint32, _P, _SZ, _P]
    L.hyb_gemv_dense_ex.restype = _I
    L.hyb_check_status.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_uint32)]
    L.hyb_check_status.restype = _I
    L.hyb_selftest_wait_timeout.argtypes = [_P, _SZ, ctypes.c_uint32, _P]
    L.hyb_selftest_wait_timeout.restype = _I
    L.hyb_spmv_noalloc.argtypes = [ctypes.POINTER(HybMatrix), _P, _I64, _P, _I64, _I, _P]
    L.hyb_spmv_noalloc.restype = _I
    L.hyb_spmv_noalloc_max_scratch_bytes.argtypes = []
    L.hyb_spmv_noalloc_max_scratch_bytes.restype = _SZ
    L.hyb_spmv_noalloc_check_status.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32)]
    L.hyb_spmv_noalloc_check_status.restype = _I
    L.hyb_plan_entries.argtypes = []
    L.hyb_plan_entries.restype = _SZ
    L.hyb_make_plan.argtypes = [ctypes.POINTER(HybMatrix), _P, _P, ctypes.POINTER(ctypes.c_int32),
                                _P]
    L.hyb_make_plan.restype = _I
    L.hyb_packed_sizes_nm.argtypes = [_I64, _I64, _I, _I, _I, _I, _P, _P, _P]
    L.hyb_packed_sizes_nm.restype = _I
    L.hyb_pack_nm.argtypes = [_I64, _I64, _I, _I, _I, _I, _P, _I64, _P, _P, _P, _P, _P, _P,
                              _SZ, _P]
    L.hyb_pack_nm.restype = _I
    L.hyb_spmm_skinny_nm.argtypes = [ctypes.POINTER(HybMatrix), _I, _I, _I, _P, _I64, _P,
                                     _I64, _I, _P, _SZ, _P]
    L.hyb_spmm_skinny_nm.restype = _I
    L.hyb_status_string.argtypes = [_I]
    L.hyb_status_string.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(status: int) -> str:
    return lib().hyb_status_string(int(status)).decode()


def _check(fn, rc):
    if rc != HYB_OK:
        raise HybError(fn, rc)


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _bits(t: torch.Tensor) -> torch.Tensor:
    """View a bf16 (or int16/uint16) tensor as its 16-bit patterns."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16)
    if t.dtype in (torch.int16, torch.uint16):
        return t
    raise TypeError(f"expected bf16 data, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# ---------------------------------------------------------------------------
# format
# ---------------------------------------------------------------------------

def packed_sizes(n: int, k: int, b1: int, b2: int, tile_map) -> tuple:
    """(n_vals, n_meta_bytes) for a host tile map (numpy/torch CPU uint8)."""
    m = np.ascontiguousarray(np.asarray(tile_map.cpu() if torch.is_tensor(tile_map)
                                        else tile_map, dtype=np.uint8).reshape(-1))
    nv, nm = _I64(), _I64()
    _check("hyb_packed_sizes", lib().hyb_packed_sizes(
        n, k, b1, b2, m.ctypes.data_as(_P), ctypes.byref(nv), ctypes.byref(nm)))
    return nv.value, nm.value


@dataclass
class Packed:
    """A packed tile-hybrid matrix on the device (tensors own the memory)."""
    n: int
    k: int
    b1: int
    b2: int
    tile_map: torch.Tensor   # uint8 [T], device
    vals: torch.Tensor       # int16 [n_vals] (bf16 bits), device
    meta: torch.Tensor       # uint8 [max(n_meta, 1)], device
    val_off: torch.Tensor    # int64 [T+1], device
    meta_off: torch.Tensor   # int64 [T+1], device
    n_vals: int
    n_meta: int
    plan: Optional[torch.Tensor] = None  # int64 work split (hyb_make_plan), host, optional
    plan_ctas: int = 0

    @property
    def num_tiles(self) -> int:
        return self.tile_map.numel()

    def struct(self) -> HybMatrix:
        return HybMatrix(self.n, self.k, self.b1, self.b2, self.num_tiles,
                         self.tile_map.data_ptr(), self.vals.data_ptr(),
                         self.meta.data_ptr(), self.val_off.data_ptr(),
                         self.meta_off.data_ptr(), self.n_vals, self.n_meta,
                         None if self.plan is None else self.plan.data_ptr(),
                         self.plan_ctas if self.plan is not None else 0)

    def nbytes(self) -> int:
        """Packed bytes the product streams (values + masks)."""
        return 2 * self.n_vals + self.n_meta

    def clone(self) -> "Packed":
        return Packed(self.n, self.k, self.b1, self.b2, self.tile_map.clone(),
                      self.vals.clone(), self.meta.clone(), self.val_off.clone(),
                      self.meta_off.clone(), self.n_vals, self.n_meta,
                      None if self.plan is None else self.plan.clone(), self.plan_ctas)


def shard_bands(n: int, k: int, b1: int, b2: int, tile_map, world: int, rank: int):
    """hyb_shard_bands: the tile-row bands [begin, end) rank `rank` of `world`
    holds (host only)."""
    tm = tile_map.cpu().numpy() if torch.is_tensor(tile_map) else np.asarray(tile_map)
    tm = np.ascontiguousarray(tm, dtype=np.uint8).reshape(-1)
    lo, hi = ctypes.c_int64(0), ctypes.c_int64(0)
    _check("hyb_shard_bands", lib().hyb_shard_bands(n, k, b1, b2, tm.ctypes.data, world, rank,
                                                    ctypes.byref(lo), ctypes.byref(hi)))
    return lo.value, hi.value


def shard(A: "Packed", rank: int, world: int, plan: bool = True) -> Optional["Packed"]:
    """The rows of A that rank `rank` of `world` holds (hyb_shard_bands): its
    bands' slice of A's packed buffers (views), offsets rebased to the slice,
    and (with ``plan``, on a GPU) its own work split.  None when the rank
    holds no band."""
    r0, r1 = shard_bands(A.n, A.k, A.b1, A.b2, A.tile_map, world, rank)
    if r1 <= r0:
        return None
    tpr = A.k // A.b2
    t0, t1 = r0 * tpr, r1 * tpr
    vo, mo = A.val_off[t0:t1 + 1], A.meta_off[t0:t1 + 1]
    v0, v1, m0, m1 = int(vo[0]), int(vo[-1]), int(mo[0]), int(mo[-1])
    # a shard without 2:4 tiles still passes a valid, aligned mask pointer
    meta = A.meta[m0:m1] if m1 > m0 else torch.zeros(16, dtype=torch.uint8, device=A.meta.device)
    S = Packed((r1 - r0) * A.b1, A.k, A.b1, A.b2, A.tile_map[t0:t1], A.vals[v0:v1], meta,
               vo - v0, mo - m0, v1 - v0, m1 - m0)
    if plan and S.val_off.is_cuda:
        S.plan, S.plan_ctas = make_plan(S)
    return S


def pack_workspace_bytes() -> int:
    return int(lib().hyb_pack_workspace_bytes())


def workspace_init(ws: torch.Tensor, stream=None):
    _check("hyb_workspace_init", lib().hyb_workspace_init(_ptr(ws), ws.numel(), _stream(stream)))


def new_workspace(nbytes: int, device) -> torch.Tensor:
    """Zeroed device workspace (uint8), 256-byte aligned by the allocator."""
    ws = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)
    assert ws.data_ptr() % 256 == 0
    return ws


def make_plan(A: "Packed", stream=None):
    """hyb_make_plan: the product's work split for A on the current device;
    returns (host int64 plan tensor, CTA count).  Synchronises the stream."""
    entries = int(lib().hyb_plan_entries())
    scratch = torch.empty(entries, dtype=torch.int64, device=A.val_off.device)
    plan = torch.zeros(entries, dtype=torch.int64)
    s = A.struct()
    s.plan = None
    ctas = ctypes.c_int32(0)
    _check("hyb_make_plan", lib().hyb_make_plan(ctypes.byref(s), _ptr(scratch), _ptr(plan),
                                                ctypes.byref(ctas), _stream(stream)))
    return plan, ctas.value


def pack(W: torch.Tensor, tile_map, b1: int, b2: int, ws: torch.Tensor = None,
         stream=None, check: bool = True, plan: bool = True) -> Packed:
    """hyb_pack: dense bf16 W [n][k] (device) + tile map -> Packed.

    With ``check`` the call synchronises and raises HybError on a NaN weight or
    a bad map byte (the pack itself is complete either way).  With ``plan`` the
    product's work split is made once here (hyb_make_plan)."""
    Wb = _bits(W)
    assert Wb.is_cuda and Wb.dim() == 2
    n, k = Wb.shape
    tm_host = tile_map.cpu().numpy() if torch.is_tensor(tile_map) else np.asarray(tile_map)
    tm_host = np.ascontiguousarray(tm_host, dtype=np.uint8).reshape(-1)
    nv, nm = packed_sizes(n, k, b1, b2, tm_host)
    dev = Wb.device
    tm = torch.from_numpy(tm_host).to(dev)
    T = tm.numel()
    vals = torch.empty(nv, dtype=torch.int16, device=dev)
    meta = torch.empty(max(nm, 1), dtype=torch.uint8, device=dev)
    vo = torch.empty(T + 1, dtype=torch.int64, device=dev)
    mo = torch.empty(T + 1, dtype=torch.int64, device=dev)
    own_ws = ws is None
    if own_ws:
        ws = new_workspace(pack_workspace_bytes(), dev)
    _check("hyb_pack", lib().hyb_pack(n, k, b1, b2, _ptr(Wb), Wb.stride(0), _ptr(tm),
                                      _ptr(vals), _ptr(meta), _ptr(vo), _ptr(mo),
                                      _ptr(ws), ws.numel(), _stream(stream)))
    if check:
        check_status(ws, stream)
    P = Packed(n, k, b1, b2, tm, vals, meta, vo, mo, nv, nm)
    if plan:
        P.plan, P.plan_ctas = make_plan(P, stream)
    return P


def packed_sizes_nm(n: int, k: int, b1: int, b2: int, nk: int, m: int, tile_map) -> tuple:
    """(n_vals, n_meta_bytes) of nk:m tiles for a host tile map."""
    mp = np.ascontiguousarray(np.asarray(tile_map.cpu() if torch.is_tensor(tile_map)
                                         else tile_map, dtype=np.uint8).reshape(-1))
    nv, nmb = _I64(), _I64()
    _check("hyb_packed_sizes_nm", lib().hyb_packed_sizes_nm(
        n, k, b1, b2, nk, m, mp.ctypes.data_as(_P), ctypes.byref(nv), ctypes.byref(nmb)))
    return nv.value, nmb.value


def pack_nm(W: torch.Tensor, tile_map, b1: int, b2: int, nk: int, m: int,
            ws: torch.Tensor = None, stream=None, check: bool = True,
            plan: bool = True) -> Packed:
    """hyb_pack_nm: dense bf16 W [n][k] (device) + tile map -> Packed with
    nk:m sparse tiles.  With ``plan``, 2:4 and 4:8 matrices (whose products run
    the streaming kernel) get their work split made once here."""
    Wb = _bits(W)
    assert Wb.is_cuda and Wb.dim() == 2
    n, k = Wb.shape
    tm_host = tile_map.cpu().numpy() if torch.is_tensor(tile_map) else np.asarray(tile_map)
    tm_host = np.ascontiguousarray(tm_host, dtype=np.uint8).reshape(-1)
    nv, nmb = packed_sizes_nm(n, k, b1, b2, nk, m, tm_host)
    dev = Wb.device
    tm = torch.from_numpy(tm_host).to(dev)
    T = tm.numel()
    vals = torch.empty(nv, dtype=torch.int16, device=dev)
    meta = torch.empty(max(nmb, 1), dtype=torch.uint8, device=dev)
    vo = torch.empty(T + 1, dtype=torch.int64, device=dev)
    mo = torch.empty(T + 1, dtype=torch.int64, device=dev)
    if ws is None:
        ws = new_workspace(pack_workspace_bytes(), dev)
    _check("hyb_pack_nm", lib().hyb_pack_nm(n, k, b1, b2, nk, m, _ptr(Wb), Wb.stride(0),
                                            _ptr(tm), _ptr(vals), _ptr(meta), _ptr(vo),
                                            _ptr(mo), _ptr(ws), ws.numel(), _stream(stream)))
    if check:
        check_status(ws, stream)
    P = Packed(n, k, b1, b2, tm, vals, meta, vo, mo, nv, nmb)
    if plan and (nk, m) in ((2, 4), (4, 8)):
        P.plan, P.plan_ctas = make_plan(P, stream)
    return P


def spmm_skinny_nm(A: Packed, X: torch.Tensor, nk: int, m: int, Y: torch.Tensor = None,
                   ydt: int = HYB_F32, ws: torch.Tensor = None, stream=None) -> torch.Tensor:
    """hyb_spmm_skinny_nm: Y[batch][n] = W_hat X for nk:m tiles; X bf16 [batch][k]."""
    Xb = _bits(X)
    if Xb.dim() == 1:
        Xb = Xb.view(1, -1)
    batch = Xb.shape[0]
    Y = _out(A.n, batch, ydt, Xb.device, Y)
    if ws is None:
        ws = new_workspace(workspace_bytes(A, batch), Xb.device)
    s = A.struct()
    _check("hyb_spmm_skinny_nm", lib().hyb_spmm_skinny_nm(
        ctypes.byref(s), nk, m, batch, _ptr(Xb), Xb.stride(0), _ptr(Y), Y.stride(0), ydt,
        _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def selftest_wait_timeout(ws: torch.Tensor, wait_limit: int = 2000, stream=None):
    """hyb_selftest_wait_timeout: launch the failure-path self test (a bounded
    wait that can never complete); the next check_status reports the timeout."""
    _check("hyb_selftest_wait_timeout",
           lib().hyb_selftest_wait_timeout(_ptr(ws), ws.numel(), wait_limit, _stream(stream)))


def check_status(ws: torch.Tensor, stream=None) -> int:
    """hyb_check_status: sync, read + clear the status word; raise on a flag."""
    flags = ctypes.c_uint32(0)
    rc = lib().hyb_check_status(_ptr(ws), _stream(stream), ctypes.byref(flags))
    if rc != HYB_OK:
        err = HybError("hyb_check_status", rc)
        err.flags = flags.value
        raise err
    return flags.value


# ---------------------------------------------------------------------------
# products
# ---------------------------------------------------------------------------

def workspace_bytes(A: Packed, batch: int = 1, rank: int = 0) -> int:
    s = A.struct()
    nbytes = int(lib().hyb_workspace_bytes(ctypes.byref(s), batch, rank))
    if nbytes == 0:
        raise HybError("hyb_workspace_bytes", HYB_ERR_INVALID_ARG)
    return nbytes


def _lowrank_struct(lowrank):
    if lowrank is None:
        return None, None
    U, V = (_bits(t) for t in lowrank)
    lr = HybLowrank(U.shape[1], U.data_ptr(), U.stride(0), V.data_ptr(), V.stride(0))
    return lr, (U, V)


def _out(n, batch, ydt, device, Y):
    if Y is not None:
        return Y
    dt = torch.float32 if ydt == HYB_F32 else torch.bfloat16
    return torch.empty(batch, n, dtype=dt, device=device)


def spmm_skinny(A: Packed, X: torch.Tensor, Y: torch.Tensor = None, ydt: int = HYB_F32,
                lowrank=None, ws: torch.Tensor = None, stream=None,
                flags: int = 0) -> torch.Tensor:
    """hyb_spmm_skinny_ex: Y[batch][n] = W_hat X (+ U (V^T X)); X bf16 [batch][k].
    flags: LAUNCH_OVERLAP_PREV lets the kernel start streaming A before the
    kernel queued ahead of it on the stream has finished (A must not be
    written by that kernel)."""
    Xb = _bits(X)
    if Xb.dim() == 1:
        Xb = Xb.view(1, -1)
    batch = Xb.shape[0]
    Y = _out(A.n, batch, ydt, Xb.device, Y)
    lr, keep = _lowrank_struct(lowrank)
    if ws is None:
        ws = new_workspace(workspace_bytes(A, batch, lr.rank if lr else 0), Xb.device)
    s = A.struct()
    _check("hyb_spmm_skinny_ex", lib().hyb_spmm_skinny_ex(
        ctypes.byref(s), batch, _ptr(Xb), Xb.stride(0), _ptr(Y), Y.stride(0), ydt,
        ctypes.byref(lr) if lr else None, flags, _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def spmm_prefill(A: Packed, X: torch.Tensor, Y: torch.Tensor = None, ws: torch.Tensor = None,
                 stream=None, block=None) -> torch.Tensor:
    """hyb_spmm_prefill: Y[m][n] = W_hat X for m tokens (tensor cores); X bf16
    [m][k], Y fp32 [m][n].  block = (rows, tokens) calls
    hyb_spmm_prefill_blocked with that CTA shape."""
    Xb = _bits(X)
    m = Xb.shape[0]
    if Y is None:
        Y = torch.empty(m, A.n, dtype=torch.float32, device=Xb.device)
    if ws is None:
        ws = new_workspace(int(lib().hyb_prefill_workspace_bytes()), Xb.device)
    s = A.struct()
    if block is None:
        _check("hyb_spmm_prefill", lib().hyb_spmm_prefill(
            ctypes.byref(s), m, _ptr(Xb), Xb.stride(0), _ptr(Y), Y.stride(0), _ptr(ws),
            ws.numel(), _stream(stream)))
    else:
        _check("hyb_spmm_prefill_blocked", lib().hyb_spmm_prefill_blocked(
            ctypes.byref(s), m, _ptr(Xb), Xb.stride(0), _ptr(Y), Y.stride(0), block[0], block[1],
            _ptr(ws), ws.numel(), _stream(stream)))
    return Y


PREFILL_SHAPES = ((128, 128), (128, 256), (256, 240), (256, 208))


def prefill_block_shape(n: int, m: int):
    """hyb_prefill_block_shape: the (rows, tokens) CTA shape hyb_spmm_prefill takes."""
    r, t = ctypes.c_int(0), ctypes.c_int(0)
    _check("hyb_prefill_block_shape",
           lib().hyb_prefill_block_shape(n, m, ctypes.byref(r), ctypes.byref(t)))
    return r.value, t.value


def gate_up_workspace_bytes(Ag: Packed, Au: Packed, batch: int, rank: int) -> int:
    sg, su = Ag.struct(), Au.struct()
    return int(lib().hyb_gate_up_workspace_bytes(ctypes.byref(sg), ctypes.byref(su), batch, rank))


def spmm_skinny_gate_up(Ag: Packed, Au: Packed, X: torch.Tensor, Ug: torch.Tensor,
                        Uu: torch.Tensor, V: torch.Tensor, ydt: int = HYB_F32,
                        ws: torch.Tensor = None, stream=None, flags: int = 0):
    """hyb_spmm_skinny_gate_up: (Yg, Yu) = (Ag X + Ug (V^T X), Au X + Uu (V^T X))
    with V^T X computed once; X bf16 [batch][k]."""
    Xb = _bits(X)
    if Xb.dim() == 1:
        Xb = Xb.view(1, -1)
    batch = Xb.shape[0]
    Yg = _out(Ag.n, batch, ydt, Xb.device, None)
    Yu = _out(Au.n, batch, ydt, Xb.device, None)
    lr, keep = _lowrank_struct((Ug, V))
    Uub = _bits(Uu)
    if ws is None:
        ws = new_workspace(gate_up_workspace_bytes(Ag, Au, batch, lr.rank), Xb.device)
    sg, su = Ag.struct(), Au.struct()
    _check("hyb_spmm_skinny_gate_up", lib().hyb_spmm_skinny_gate_up(
        ctypes.byref(sg), ctypes.byref(su), batch, _ptr(Xb), Xb.stride(0), _ptr(Yg),
        Yg.stride(0), _ptr(Yu), Yu.stride(0), ydt, ctypes.byref(lr), _ptr(Uub), Uub.stride(0),
        flags, _ptr(ws), ws.numel(), _stream(stream)))
    return Yg, Yu


def spmv(A: Packed, x: torch.Tensor, y: torch.Tensor = None, ydt: int = HYB_F32,
         lowrank=None, ws: torch.Tensor = None, stream=None) -> torch.Tensor:
    """hyb_spmv: y[1][n] = W_hat x (+ U (V^T x)); x bf16 [k] or [1][k]."""
    xb = _bits(x).reshape(1, -1)
    y = _out(A.n, 1, ydt, xb.device, y)
    lr, keep = _lowrank_struct(lowrank)
    if ws is None:
        ws = new_workspace(workspace_bytes(A, 1, lr.rank if lr else 0), xb.device)
    s = A.struct()
    _check("hyb_spmv", lib().hyb_spmv(
        ctypes.byref(s), _ptr(xb), xb.stride(0), _ptr(y), y.stride(0), ydt,
        ctypes.byref(lr) if lr else None, _ptr(ws), ws.numel(), _stream(stream)))
    return y


def lowrank_workspace_bytes(k: int, batch: int, rank: int) -> int:
    return int(lib().hyb_lowrank_workspace_bytes(k, batch, rank))


def lowrank_add(U: torch.Tensor, V: torch.Tensor, X: torch.Tensor, Y: torch.Tensor,
                ws: torch.Tensor = None, stream=None) -> torch.Tensor:
    """hyb_lowrank_add: Y (fp32 [batch][n]) += U (V^T X), in place."""
    Xb = _bits(X)
    if Xb.dim() == 1:
        Xb = Xb.view(1, -1)
    batch, k = Xb.shape
    n = Y.shape[-1]
    lr, keep = _lowrank_struct((U, V))
    if ws is None:
        ws = new_workspace(lowrank_workspace_bytes(k, batch, lr.rank), Xb.device)
    _check("hyb_lowrank_add", lib().hyb_lowrank_add(
        n, k, batch, ctypes.byref(lr), _ptr(Xb), Xb.stride(0), _ptr(Y), Y.stride(0),
        _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def dense_workspace_bytes(n: int, k: int, batch: int = 1) -> int:
    return int(lib().hyb_dense_workspace_bytes(n, k, batch))


def gemv_dense(W: torch.Tensor, X: torch.Tensor, Y: torch.Tensor = None,
               ydt: int = HYB_F32, ws: torch.Tensor = None, stream=None,
               flags: int = 0) -> torch.Tensor:
    """hyb_gemv_dense_ex: Y[batch][n] = W X for a plain row-major bf16 W [n][k]
    (flags as for spmm_skinny)."""
    Wb = _bits(W)
    Xb = _bits(X)
    if Xb.dim() == 1:
        Xb = Xb.view(1, -1)
    n, k = Wb.shape
    batch = Xb.shape[0]
    Y = _out(n, batch, ydt, Xb.device, Y)
    if ws is None:
        ws = new_workspace(dense_workspace_bytes(n, k, batch), Xb.device)
    _check("hyb_gemv_dense_ex", lib().hyb_gemv_dense_ex(
        n, k, batch, _ptr(Wb), Wb.stride(0), _ptr(Xb), Xb.stride(0), _ptr(Y), Y.stride(0),
        ydt, flags, _ptr(ws), ws.numel(), _stream(stream)))
    return Y


def spmv_noalloc(A: Packed, x: torch.Tensor, y: torch.Tensor = None, ydt: int = HYB_F32,
                 stream=None) -> torch.Tensor:
    """hyb_spmv_noalloc: hyb_spmv (batch 1, no low-rank term) without a caller
    workspace; the library's own static device array holds the scratch, so the
    call allocates nothing (``y`` may be passed in to avoid the output
    allocation here too).  Make the first call on a device outside any stream
    capture, and do not let two calls overlap on the GPU."""
    xb = _bits(x).reshape(1, -1)
    y = _out(A.n, 1, ydt, xb.device, y)
    s = A.struct()
    _check("hyb_spmv_noalloc", lib().hyb_spmv_noalloc(
        ctypes.byref(s), _ptr(xb), xb.stride(0), _ptr(y), y.stride(0), ydt, _stream(stream)))
    return y


def spmv_noalloc_max_scratch_bytes() -> int:
    return int(lib().hyb_spmv_noalloc_max_scratch_bytes())


def spmv_noalloc_check_status(stream=None) -> int:
    """hyb_spmv_noalloc_check_status: sync, read + clear the status word of the
    static array behind hyb_spmv_noalloc; raise on a flag."""
    flags = ctypes.c_uint32(0)
    rc = lib().hyb_spmv_noalloc_check_status(_stream(stream), ctypes.byref(flags))
    if rc != HYB_OK:
        err = HybError("hyb_spmv_noalloc_check_status", rc)
        err.flags = flags.value
        raise err
    return flags.value
