"""B200-native weight-only skinny GEMM: y[M,N] = x[M,K] . W^T, M = 1..16,
with W kept in HBM as NVFP4 (E2M1 codes + UE4M3 per-16 scales + FP32 global)
or FP8 E4M3 (+ FP32 per output channel), FP16 activations, FP32 accumulation.

This module is a thin ctypes binding over ``libskinny.so`` (whose C ABI is
``include/skinny.h``): it turns numpy arrays and torch tensors into pointers,
sizes and a stream handle, calls the library, and raises ``SkinnyError`` on a
non-zero status.  Every step of the GEMM runs in the library's CUDA kernels;
there is no fallback: if the library is missing, the first call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import threading

import numpy as np

_PKG = os.path.dirname(os.path.abspath(__file__))
LIBRARY_PATH = os.path.join(_PKG, "libskinny.so")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_ALIGNMENT = -3
ERR_CUDA = -4
ERR_WORKSPACE = -5

OUT_F16 = 0
OUT_F32 = 1
FMT_NVFP4 = 0
FMT_FP8 = 1
MAX_M = 16
MAX_GROUP = 8

_lock = threading.Lock()
_lib = None


class GroupMember(ctypes.Structure):
    """skinny_nvfp4_group_member of include/skinny.h."""
    _fields_ = [("x", ctypes.c_void_p), ("w_packed", ctypes.c_void_p), ("global_scale", ctypes.c_float),
                ("N", ctypes.c_int64), ("y", ctypes.c_void_p)]


class SkinnyError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__("%s: %s (%d)" % (what, status_string(status), status))


def library() -> ctypes.CDLL:
    """Load libskinny.so (built by ``__graft_entry__.build()``); raise if absent."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIBRARY_PATH):
                raise RuntimeError("libskinny.so is not built (%s); run __graft_entry__.build()" % LIBRARY_PATH)
            lib = ctypes.CDLL(LIBRARY_PATH)
            p, i64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t
            sigs = {
                "skinny_status_string": (ctypes.c_char_p, [ctypes.c_int]),
                "skinny_version": (ctypes.c_int, []),
                "skinny_nvfp4_packed_bytes": (sz, [i64, i64]),
                "skinny_pack_nvfp4": (ctypes.c_int, [p, p, i64, i64, p]),
                "skinny_unpack_nvfp4": (ctypes.c_int, [p, i64, i64, p, p]),
                "skinny_fp8_packed_bytes": (sz, [i64, i64]),
                "skinny_pack_fp8": (ctypes.c_int, [p, i64, i64, p]),
                "skinny_unpack_fp8": (ctypes.c_int, [p, i64, i64, p]),
                "skinny_workspace_bytes": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, i64, i64, ctypes.POINTER(sz)]),
                "skinny_nvfp4_gemm": (ctypes.c_int, [p, ctypes.c_int, i64, p, ctypes.c_float, i64, p, ctypes.c_int,
                                                     p, sz, p]),
                "skinny_fp8_gemm": (ctypes.c_int, [p, ctypes.c_int, i64, p, p, i64, p, ctypes.c_int, p, sz, p]),
                "skinny_device_error": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_uint)]),
                "skinny_nvfp4_gemm_static_ws": (ctypes.c_int, [p, ctypes.c_int, i64, p, ctypes.c_float, i64, p,
                                                               ctypes.c_int, p]),
                "skinny_nvfp4_gemm_argmax": (ctypes.c_int, [p, ctypes.c_int, i64, p, ctypes.c_float, i64, p, p, p,
                                                            sz, p]),
                "skinny_pack_nvfp4_gate_up": (ctypes.c_int, [p, p, i64, i64, p]),
                "skinny_debug_schedule": (ctypes.c_int, [i64, i64, ctypes.c_int, ctypes.c_int, p, ctypes.c_int,
                                                         ctypes.POINTER(ctypes.c_int)]),
                "skinny_nvfp4_gemm_add": (ctypes.c_int, [p, ctypes.c_int, i64, p, ctypes.c_float, i64, p, p,
                                                         ctypes.c_int, p, sz, p]),
                "skinny_fp8_gemm_add": (ctypes.c_int, [p, ctypes.c_int, i64, p, p, i64, p, p, ctypes.c_int, p, sz,
                                                       p]),
                "skinny_nvfp4_gemm_silu_mul": (ctypes.c_int, [p, ctypes.c_int, i64, p, ctypes.c_float, i64, p,
                                                              ctypes.c_int, p, sz, p]),
                "skinny_static_workspace_capacity": (sz, []),
                "skinny_stream_read": (ctypes.c_int, [p, sz, ctypes.c_int, p, p]),
                "skinny_nvfp4_gemm_grouped": (ctypes.c_int, [ctypes.POINTER(GroupMember), ctypes.c_int,
                                                             ctypes.c_int, i64, ctypes.c_int, p, sz, p]),
                "skinny_debug_static_workspace_address": (ctypes.c_int, [ctypes.POINTER(ctypes.c_void_p)]),
            }
            for name, (res, args) in sigs.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().skinny_status_string(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise SkinnyError(status, what)


def _np_ptr(a: np.ndarray) -> int:
    return a.ctypes.data


# ---------------------------------------------------------------------------
# Host-side packing
# ---------------------------------------------------------------------------

def nvfp4_packed_bytes(N: int, K: int) -> int:
    """Bytes of the packed NVFP4 layout (codes and block scales)."""
    return int(library().skinny_nvfp4_packed_bytes(int(N), int(K)))


def fp8_packed_bytes(N: int, K: int) -> int:
    return int(library().skinny_fp8_packed_bytes(int(N), int(K)))


def pack_nvfp4(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Logical codes [N, K/2] (low nibble = even k) and UE4M3 scales [N, K/16] ->
    the packed uint8 buffer (tiles of codes with their block scales)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    N, K = codes.shape[0], codes.shape[1] * 2
    if scales.shape != (N, K // 16):
        raise ValueError("scales must be [N, K/16]")
    nb = nvfp4_packed_bytes(N, K)
    if nb == 0:
        raise SkinnyError(ERR_INVALID_ARG, "pack_nvfp4 shape")
    out = np.empty(nb, np.uint8)
    _check(library().skinny_pack_nvfp4(_np_ptr(codes), _np_ptr(scales), N, K, _np_ptr(out)), "skinny_pack_nvfp4")
    return out


def unpack_nvfp4(packed: np.ndarray, N: int, K: int):
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    codes, scales = np.empty((N, K // 2), np.uint8), np.empty((N, K // 16), np.uint8)
    _check(library().skinny_unpack_nvfp4(_np_ptr(packed), N, K, _np_ptr(codes), _np_ptr(scales)),
           "skinny_unpack_nvfp4")
    return codes, scales


def pack_fp8(q: np.ndarray) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.uint8)
    N, K = q.shape
    nb = fp8_packed_bytes(N, K)
    if nb == 0:
        raise SkinnyError(ERR_INVALID_ARG, "pack_fp8 shape")
    out = np.empty(nb, np.uint8)
    _check(library().skinny_pack_fp8(_np_ptr(q), N, K, _np_ptr(out)), "skinny_pack_fp8")
    return out


def unpack_fp8(packed: np.ndarray, N: int, K: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    q = np.empty((N, K), np.uint8)
    _check(library().skinny_unpack_fp8(_np_ptr(packed), N, K, _np_ptr(q)), "skinny_unpack_fp8")
    return q


# ---------------------------------------------------------------------------
# Device GEMMs (torch supplies device memory and the stream)
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class PackedNVFP4:
    data: "object"           # torch.uint8 device tensor (packed tiles: codes + block scales)
    global_scale: float
    N: int
    K: int

    @classmethod
    def from_logical(cls, codes: np.ndarray, scales: np.ndarray, global_scale: float, device="cuda"):
        import torch

        return cls(torch.from_numpy(pack_nvfp4(codes, scales)).to(device), float(global_scale), codes.shape[0],
                   codes.shape[1] * 2)

    @property
    def fmt(self) -> int:
        return FMT_NVFP4

    @property
    def nbytes(self) -> int:
        return int(self.data.numel())


@dataclasses.dataclass
class PackedFP8:
    codes: "object"          # torch.uint8 device tensor (packed layout)
    channel_scale: "object"  # torch.float32 device tensor [N]
    N: int
    K: int

    @classmethod
    def from_logical(cls, q: np.ndarray, channel_scale: np.ndarray, device="cuda"):
        import torch

        return cls(torch.from_numpy(pack_fp8(q)).to(device),
                   torch.from_numpy(np.ascontiguousarray(channel_scale, np.float32)).to(device), q.shape[0], q.shape[1])

    @property
    def fmt(self) -> int:
        return FMT_FP8

    @property
    def nbytes(self) -> int:
        return int(self.codes.numel() + 4 * self.channel_scale.numel())


def workspace_bytes(fmt: int, M: int, N: int, K: int) -> int:
    """Split-K workspace size for one GEMM on the current device."""
    b = ctypes.c_size_t(0)
    _check(library().skinny_workspace_bytes(int(fmt), int(M), int(N), int(K), ctypes.byref(b)),
           "skinny_workspace_bytes")
    return int(b.value)


def make_workspace(fmt: int, M: int, N: int, K: int, device="cuda"):
    """A zero-filled workspace (its partial-sum slots must start at zero)."""
    import torch

    return torch.zeros(workspace_bytes(fmt, M, N, K), dtype=torch.uint8, device=device)


def _stream_handle(stream) -> int:
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def gemm_into(y, x, w, workspace=None, stream=None) -> None:
    """y[M, N] = x[M, K] . W^T on the device (y float16 or float32, preallocated)."""
    import torch

    M, K = x.shape
    if x.dtype != torch.float16 or not x.is_contiguous() or K != w.K:
        raise ValueError("x must be a contiguous float16 [M, %d] tensor" % w.K)
    if y.shape != (M, w.N) or not y.is_contiguous() or y.dtype not in (torch.float16, torch.float32):
        raise ValueError("y must be a contiguous float16/float32 [M, N] tensor")
    out = OUT_F32 if y.dtype == torch.float32 else OUT_F16
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    h = _stream_handle(stream)
    lib = library()
    if w.fmt == FMT_NVFP4:
        st = lib.skinny_nvfp4_gemm(x.data_ptr(), M, K, w.data.data_ptr(), ctypes.c_float(w.global_scale), w.N,
                                   y.data_ptr(), out, ws_ptr, ws_bytes, h)
        _check(st, "skinny_nvfp4_gemm")
    else:
        st = lib.skinny_fp8_gemm(x.data_ptr(), M, K, w.codes.data_ptr(), w.channel_scale.data_ptr(), w.N,
                                 y.data_ptr(), out, ws_ptr, ws_bytes, h)
        _check(st, "skinny_fp8_gemm")


def gemm_add_into(y, x, w, residual, workspace=None, stream=None) -> None:
    """y[M, N] = x . W^T + residual, the add in FP32 before the one output
    rounding; residual has y's shape and dtype and may be y itself."""
    import torch

    M, K = x.shape
    if x.dtype != torch.float16 or not x.is_contiguous() or K != w.K:
        raise ValueError("x must be a contiguous float16 [M, %d] tensor" % w.K)
    if y.shape != (M, w.N) or not y.is_contiguous() or y.dtype not in (torch.float16, torch.float32):
        raise ValueError("y must be a contiguous float16/float32 [M, N] tensor")
    if residual.shape != y.shape or residual.dtype != y.dtype or not residual.is_contiguous():
        raise ValueError("residual must be a contiguous tensor of y's shape and dtype")
    out = OUT_F32 if y.dtype == torch.float32 else OUT_F16
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    h = _stream_handle(stream)
    lib = library()
    if w.fmt == FMT_NVFP4:
        st = lib.skinny_nvfp4_gemm_add(x.data_ptr(), M, K, w.data.data_ptr(), ctypes.c_float(w.global_scale), w.N,
                                       residual.data_ptr(), y.data_ptr(), out, ws_ptr, ws_bytes, h)
        _check(st, "skinny_nvfp4_gemm_add")
    else:
        st = lib.skinny_fp8_gemm_add(x.data_ptr(), M, K, w.codes.data_ptr(), w.channel_scale.data_ptr(), w.N,
                                     residual.data_ptr(), y.data_ptr(), out, ws_ptr, ws_bytes, h)
        _check(st, "skinny_fp8_gemm_add")


def gemm_grouped_into(ys, xs, ws, workspace=None, stream=None) -> None:
    """ys[i][M, N_i] = xs[i][M, K] . W_i^T for every i, in ONE launch (NVFP4
    weights of the same K; ys all float16 or all float32, preallocated)."""
    import torch

    if not (len(ys) == len(xs) == len(ws)) or not 1 <= len(ws) <= MAX_GROUP:
        raise ValueError("ys, xs and ws must have the same length, 1..%d" % MAX_GROUP)
    M, K = xs[0].shape
    dt = ys[0].dtype
    members = (GroupMember * len(ws))()
    for i, (y, x, w) in enumerate(zip(ys, xs, ws)):
        if w.fmt != FMT_NVFP4 or w.K != K:
            raise ValueError("grouped GEMMs take NVFP4 weights of one K")
        if x.dtype != torch.float16 or not x.is_contiguous() or x.shape != (M, K):
            raise ValueError("every x must be a contiguous float16 [%d, %d] tensor" % (M, K))
        if y.shape != (M, w.N) or not y.is_contiguous() or y.dtype != dt or dt not in (torch.float16, torch.float32):
            raise ValueError("every y must be a contiguous [M, N_i] tensor of one dtype (float16 or float32)")
        members[i] = GroupMember(x.data_ptr(), w.data.data_ptr(), w.global_scale, w.N, y.data_ptr())
    out = OUT_F32 if dt == torch.float32 else OUT_F16
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = library().skinny_nvfp4_gemm_grouped(members, len(ws), M, K, out, ws_ptr, ws_bytes, _stream_handle(stream))
    _check(st, "skinny_nvfp4_gemm_grouped")


def gemm(x, w, out_dtype=None, workspace=None, stream=None):
    """Allocate y and compute y = x . W^T (float16 output unless out_dtype says otherwise)."""
    import torch

    y = torch.empty((x.shape[0], w.N), dtype=out_dtype or torch.float16, device=x.device)
    gemm_into(y, x, w, workspace=workspace, stream=stream)
    return y


def pack_nvfp4_gate_up(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Pack gate+up weights (rows 0..F-1 gate, F..2F-1 up) for the fused SiLU*mul GEMM."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    n2, half_k = codes.shape
    K = 2 * half_k
    if n2 % 2 or scales.shape != (n2, K // 16):
        raise ValueError("codes [2F, K/2] and scales [2F, K/16] expected")
    out = np.zeros(nvfp4_packed_bytes(n2, K), np.uint8)
    _check(library().skinny_pack_nvfp4_gate_up(codes.ctypes.data, scales.ctypes.data, n2 // 2, K, out.ctypes.data),
           "skinny_pack_nvfp4_gate_up")
    return out


@dataclasses.dataclass
class PackedGateUp:
    """Gate+up NVFP4 weights packed for gemm_silu_mul: F outputs, 2F weight rows."""
    data: "object"
    global_scale: float
    F: int
    K: int

    @classmethod
    def from_logical(cls, codes: np.ndarray, scales: np.ndarray, global_scale: float, device="cuda"):
        import torch

        return cls(torch.from_numpy(pack_nvfp4_gate_up(codes, scales)).to(device), float(global_scale),
                   codes.shape[0] // 2, codes.shape[1] * 2)

    @property
    def fmt(self) -> int:
        return FMT_NVFP4

    @property
    def N(self) -> int:
        """Weight rows (gate and up): the GEMM's N, e.g. for workspace_bytes."""
        return 2 * self.F


def gemm_silu_mul_into(y, x, w: "PackedGateUp", workspace=None, stream=None) -> None:
    """y[M, F] = silu(x . Wgate^T) * (x . Wup^T) (y float16 or float32, preallocated)."""
    import torch

    if not isinstance(w, PackedGateUp):
        raise TypeError("gemm_silu_mul takes weights packed by PackedGateUp / pack_nvfp4_gate_up")
    M, K = x.shape
    if x.dtype != torch.float16 or not x.is_contiguous() or K != w.K:
        raise ValueError("x must be a contiguous float16 [M, %d] tensor" % w.K)
    if y.shape != (M, w.F) or not y.is_contiguous() or y.dtype not in (torch.float16, torch.float32):
        raise ValueError("y must be a contiguous float16/float32 [M, F] tensor")
    out = OUT_F32 if y.dtype == torch.float32 else OUT_F16
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = library().skinny_nvfp4_gemm_silu_mul(x.data_ptr(), M, K, w.data.data_ptr(), ctypes.c_float(w.global_scale),
                                              w.F, y.data_ptr(), out, ws_ptr, ws_bytes, _stream_handle(stream))
    _check(st, "skinny_nvfp4_gemm_silu_mul")


def gemm_silu_mul(x, w: "PackedGateUp", out_dtype=None, workspace=None, stream=None):
    """Allocate y [M, F] and compute the fused gate+up GEMM with SiLU*mul."""
    import torch

    y = torch.empty((x.shape[0], w.F), dtype=out_dtype or torch.float16, device=x.device)
    gemm_silu_mul_into(y, x, w, workspace=workspace, stream=stream)
    return y


def gemm_argmax_into(idx, val, x, w, workspace, stream=None) -> None:
    """Per token m: idx[m] = argmax_n y[m, n], val[m] = y[m, idx[m]] for y = x . W^T
    (NVFP4 W), without writing y.  idx int32 [M], val float32 [M]; the workspace
    (zero-filled, from make_workspace) is required."""
    import torch

    M, K = x.shape
    if x.dtype != torch.float16 or not x.is_contiguous() or K != w.K:
        raise ValueError("x must be a contiguous float16 [M, %d] tensor" % w.K)
    if w.fmt != FMT_NVFP4:
        raise ValueError("the fused argmax takes NVFP4 weights")
    if idx.shape != (M,) or idx.dtype != torch.int32 or val.shape != (M,) or val.dtype != torch.float32:
        raise ValueError("idx must be int32 [M] and val float32 [M]")
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = library().skinny_nvfp4_gemm_argmax(x.data_ptr(), M, K, w.data.data_ptr(), ctypes.c_float(w.global_scale),
                                            w.N, idx.data_ptr(), val.data_ptr(), ws_ptr, ws_bytes,
                                            _stream_handle(stream))
    _check(st, "skinny_nvfp4_gemm_argmax")


def gemm_argmax(x, w, workspace, stream=None):
    """Allocate and return (idx int32 [M], val float32 [M]): see gemm_argmax_into."""
    import torch

    idx = torch.empty((x.shape[0],), dtype=torch.int32, device=x.device)
    val = torch.empty((x.shape[0],), dtype=torch.float32, device=x.device)
    gemm_argmax_into(idx, val, x, w, workspace, stream=stream)
    return idx, val


def device_error(clear: bool = True) -> int:
    """Synchronise and read the device-side error word (0 = no wait gave up)."""
    v = ctypes.c_uint(0)
    _check(library().skinny_device_error(1 if clear else 0, ctypes.byref(v)), "skinny_device_error")
    return int(v.value)
