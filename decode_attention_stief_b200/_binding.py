"""ctypes binding of libstief.so: argument marshalling only.

Every function here takes torch tensors, checks dtype / device / contiguity /
shape agreement, and passes raw device pointers, sizes and the current CUDA
stream to the C entry point of the same name.  All arithmetic runs in the
library's CUDA kernels.  There is no fallback path: a missing or unloadable
library raises ``StiefError``.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.environ.get("STIEF_LIBRARY", os.path.join(_PKG, "libstief.so"))

STATUS = {
    0: "STIEF_OK",
    1: "STIEF_ERR_INVALID_ARG",
    2: "STIEF_ERR_ALIGNMENT",
    3: "STIEF_ERR_CAPACITY",
    4: "STIEF_ERR_WORKSPACE",
    5: "STIEF_ERR_CUDA",
    6: "STIEF_ERR_DEVICE_STATUS",
    7: "STIEF_ERR_UNSUPPORTED_DEVICE",
}
DEV_CAPACITY_OVERFLOW = 0x1
DEV_WAIT_TIMEOUT = 0x2
DEV_BAD_LENGTH = 0x4


class StiefError(RuntimeError):
    """A libstief call returned a non-OK status (or the library is missing)."""

    def __init__(self, func: str, code: int):
        self.code = code
        super().__init__(f"{func}: {STATUS.get(code, code)}")


_lock = threading.Lock()
_lib = None

_u16p = ctypes.c_void_p
_i = ctypes.c_int


def library_path() -> str:
    return _LIB_PATH


def library() -> ctypes.CDLL:
    """Load libstief.so (once).  Raises StiefError if it is missing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise StiefError(f"libstief.so not found at {_LIB_PATH}; build it with "
                                 "python -m decode_attention_stief_b200.build", -1)
            lib = ctypes.CDLL(_LIB_PATH)
            vp = ctypes.c_void_p
            lib.stief_compress_append.restype = _i
            lib.stief_compress_append.argtypes = [vp] * 7 + [_i] * 7 + [vp, vp]
            lib.stief_decode_attention.restype = _i
            lib.stief_decode_attention.argtypes = ([vp] * 8 + [ctypes.c_size_t] + [_i] * 9
                                                   + [vp, vp])
            lib.stief_decode_workspace_bytes.restype = ctypes.c_size_t
            lib.stief_decode_workspace_bytes.argtypes = [_i] * 5
            lib.stief_decode_max_splits.restype = _i
            lib.stief_decode_max_splits.argtypes = [_i]
            lib.stief_decode_auto_splits.restype = _i
            lib.stief_decode_auto_splits.argtypes = [_i] * 5
            lib.stief_append_decode.restype = _i
            lib.stief_append_decode.argtypes = ([vp] * 10 + [ctypes.c_size_t] + [_i] * 9
                                                + [vp, vp])
            lib.stief_compress_append_paged.restype = _i
            lib.stief_compress_append_paged.argtypes = [vp] * 8 + [_i] * 9 + [vp, vp]
            lib.stief_decode_attention_paged.restype = _i
            lib.stief_decode_attention_paged.argtypes = ([vp] * 9 + [ctypes.c_size_t] + [_i] * 11
                                                         + [vp, vp])
            lib.stief_append_decode_paged.restype = _i
            lib.stief_append_decode_paged.argtypes = ([vp] * 11 + [ctypes.c_size_t] + [_i] * 11
                                                      + [vp, vp])
            lib.stief_compress_append_q8.restype = _i
            lib.stief_compress_append_q8.argtypes = [vp] * 9 + [_i] * 7 + [vp, vp]
            lib.stief_decode_attention_q8.restype = _i
            lib.stief_decode_attention_q8.argtypes = ([vp] * 10 + [ctypes.c_size_t] + [_i] * 9
                                                      + [vp, vp])
            lib.stief_append_decode_q8.restype = _i
            lib.stief_append_decode_q8.argtypes = ([vp] * 12 + [ctypes.c_size_t] + [_i] * 9
                                                   + [vp, vp])
            lib.stief_compress_append_q8_paged.restype = _i
            lib.stief_compress_append_q8_paged.argtypes = [vp] * 10 + [_i] * 9 + [vp, vp]
            lib.stief_decode_attention_q8_paged.restype = _i
            lib.stief_decode_attention_q8_paged.argtypes = ([vp] * 11 + [ctypes.c_size_t] + [_i] * 11
                                                            + [vp, vp])
            lib.stief_compress_append_q4.restype = _i
            lib.stief_compress_append_q4.argtypes = [vp] * 9 + [_i] * 7 + [vp, vp]
            lib.stief_decode_attention_q4.restype = _i
            lib.stief_decode_attention_q4.argtypes = ([vp] * 10 + [ctypes.c_size_t] + [_i] * 9
                                                      + [vp, vp])
            lib.stief_compress_append_joint_v.restype = _i
            lib.stief_compress_append_joint_v.argtypes = [vp] * 7 + [_i] * 7 + [vp, vp]
            lib.stief_decode_attention_joint_v.restype = _i
            lib.stief_decode_attention_joint_v.argtypes = ([vp] * 8 + [ctypes.c_size_t] + [_i] * 9
                                                           + [vp, vp])
            lib.stief_decode_latent_joint_v.restype = _i
            lib.stief_decode_latent_joint_v.argtypes = ([vp] * 6 + [ctypes.c_size_t] + [_i] * 9
                                                        + [vp, vp])
            lib.stief_decode_latent.restype = _i
            lib.stief_decode_latent.argtypes = ([vp] * 6 + [ctypes.c_size_t] + [_i] * 9
                                                + [vp, vp])
            lib.stief_decode_attention_noalloc.restype = _i
            lib.stief_decode_attention_noalloc.argtypes = [vp] * 7 + [_i] * 9 + [vp, vp]
            lib.stief_read_device_status.restype = _i
            lib.stief_read_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), vp]
            lib.stief_status_string.restype = ctypes.c_char_p
            lib.stief_status_string.argtypes = [_i]
            _lib = lib
    return _lib


def _check(func: str, code: int) -> None:
    if code != 0:
        raise StiefError(func, code)



class Prepared:
    """A library call validated once (see prepare): calling it launches the same call again with
    the same device pointers, sizes and stream, at the C call's own host cost.  It keeps the
    argument tensors alive; their storage, shapes and contents-to-be are the caller's to keep
    as they were when it was prepared (in-place updates of their values are what it is for)."""

    __slots__ = ("name", "_fn", "_cargs", "_keep")

    def __init__(self, name, cargs, keep):
        self.name = name
        self._fn = getattr(library(), name)
        self._cargs = cargs
        self._keep = keep

    def __call__(self):
        code = self._fn(*self._cargs)
        if code != 0:
            raise StiefError(self.name, code)


_capture = threading.local()


def _invoke(name: str, cargs: tuple) -> None:
    """Calls the library entry point `name` with the marshalled arguments, or, while prepare()
    is capturing, records them instead."""
    if getattr(_capture, "calls", None) is not None:
        _capture.calls.append((name, cargs))
        return
    _check(name, getattr(library(), name)(*cargs))


def prepare(fn, *args, **kwargs) -> Prepared:
    """Validates and marshals the arguments of the binding function `fn` (e.g.
    stief_append_decode) exactly as calling it would, without launching anything, and returns
    a Prepared call: a serving loop that reuses the same buffers every step calls that object
    instead, skipping the per-call checks (the library still validates sizes on every call).
    The stream is the one given, or the current stream at preparation."""
    _capture.calls = []
    try:
        fn(*args, **kwargs)
        calls = _capture.calls
    finally:
        _capture.calls = None
    if len(calls) != 1:
        raise ValueError(f"{getattr(fn, '__name__', fn)} makes {len(calls)} library calls; prepare takes one")
    name, cargs = calls[0]
    return Prepared(name, cargs, (args, kwargs))

def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dev(t: torch.Tensor, name: str, dtype: torch.dtype, ndim: int) -> int:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _opt_status(dev_status: Optional[torch.Tensor]) -> Optional[int]:
    if dev_status is None:
        return None
    if dev_status.dtype not in (torch.int32, torch.uint32) or dev_status.numel() < 1 or not dev_status.is_cuda:
        raise ValueError("dev_status must be a CUDA int32/uint32 tensor with at least one element")
    return dev_status.data_ptr()


def stief_status_string(code: int) -> str:
    return library().stief_status_string(int(code)).decode()


def stief_decode_max_splits(max_seq_len: int) -> int:
    return int(library().stief_decode_max_splits(int(max_seq_len)))


def stief_decode_auto_splits(B: int, Hq: int, Hkv: int, max_seq_len: int, num_sms: int) -> int:
    return int(library().stief_decode_auto_splits(B, Hq, Hkv, max_seq_len, num_sms))


def stief_decode_workspace_bytes(B: int, Hq: int, Hkv: int, rV: int, max_seq_len: int) -> int:
    return int(library().stief_decode_workspace_bytes(B, Hq, Hkv, rV, max_seq_len))


def workspace_for(B: int, Hq: int, Hkv: int, rV: int, max_seq_len: int,
                  device="cuda") -> torch.Tensor:
    """A zero-filled uint8 device tensor of stief_decode_workspace_bytes(...) bytes.

    Zero-filled once here; every completed decode call leaves its ticket counters at
    zero, so the tensor can be reused for any later call on the same stream.
    """
    n = stief_decode_workspace_bytes(B, Hq, Hkv, rV, max_seq_len)
    if n == 0:
        raise ValueError("invalid sizes for the decode workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def stief_compress_append(k_new: torch.Tensor, v_new: torch.Tensor, P_K: torch.Tensor,
                          P_V: torch.Tensor, k_lat: torch.Tensor, v_lat: torch.Tensor,
                          seq_lens: torch.Tensor, dev_status: Optional[torch.Tensor] = None,
                          stream=None) -> None:
    """Project T new rows per (sequence, KV head) into the latent cache and advance seq_lens.

    k_new, v_new [B][Hkv][T][d] bf16; P_K [Hkv][d][rK], P_V [Hkv][d][rV] bf16;
    k_lat [B][Hkv][L_max][rK], v_lat [B][Hkv][L_max][rV] bf16; seq_lens [B] int32.
    """
    pk = _dev(k_new, "k_new", torch.bfloat16, 4)
    pv = _dev(v_new, "v_new", torch.bfloat16, 4)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkl = _dev(k_lat, "k_lat", torch.bfloat16, 4)
    pvl = _dev(v_lat, "v_lat", torch.bfloat16, 4)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    B, Hkv, T, d = k_new.shape
    rK, rV = P_K.shape[2], P_V.shape[2]
    L_max = k_lat.shape[2]
    if tuple(v_new.shape) != (B, Hkv, T, d) or tuple(P_K.shape) != (Hkv, d, rK) \
            or tuple(P_V.shape) != (Hkv, d, rV) or tuple(k_lat.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_lat.shape) != (B, Hkv, L_max, rV) or seq_lens.shape[0] != B:
        raise ValueError("stief_compress_append: inconsistent shapes")
    _invoke("stief_compress_append", (pk, pv, ppk, ppv, pkl, pvl, psl, B, Hkv, T, d, rK,
                                           rV, L_max, _opt_status(dev_status),
                                           _stream_ptr(stream),))


def stief_decode_attention(q: torch.Tensor, P_K: torch.Tensor, P_V: torch.Tensor,
                           k_lat: torch.Tensor, v_lat: torch.Tensor, seq_lens: torch.Tensor,
                           out: torch.Tensor, workspace: torch.Tensor, max_seq_len: int,
                           num_splits: int = 0, dev_status: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """One decode step: out [B][Hq][d] = softmax(q K~^T / sqrt(d)) V~ over the latent cache.

    q [B][Hq][d] bf16; P_K [Hkv][d][rK], P_V [Hkv][d][rV] bf16;
    k_lat [B][Hkv][L_max][rK], v_lat [B][Hkv][L_max][rV] bf16; seq_lens [B] int32;
    out [B][Hq][d] bf16 (written); workspace: uint8 device tensor of at least
    stief_decode_workspace_bytes(...) bytes.
    """
    pq = _dev(q, "q", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkl = _dev(k_lat, "k_lat", torch.bfloat16, 4)
    pvl = _dev(v_lat, "v_lat", torch.bfloat16, 4)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_V.shape[2]
    L_max = k_lat.shape[2]
    if tuple(P_K.shape) != (Hkv, d, rK) or tuple(P_V.shape) != (Hkv, d, rV) \
            or tuple(k_lat.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_lat.shape) != (B, Hkv, L_max, rV) or seq_lens.shape[0] != B \
            or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_decode_attention: inconsistent shapes")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_decode_attention", (pq, ppk, ppv, pkl, pvl, psl, po,
                                            workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d, rK,
                                            rV, L_max, int(max_seq_len), int(num_splits),
                                            _opt_status(dev_status), _stream_ptr(stream),))
    return out


def stief_append_decode(q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                        P_K: torch.Tensor, P_V: torch.Tensor, k_lat: torch.Tensor,
                        v_lat: torch.Tensor, seq_lens: torch.Tensor, out: torch.Tensor,
                        workspace: torch.Tensor, max_seq_len: int, num_splits: int = 0,
                        dev_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """One whole decode step in one kernel: append the new token's compressed key and value
    rows (k_new P_K, v_new P_V at row seq_lens[b]), attend over the grown cache, and
    increment seq_lens.

    q [B][Hq][d] bf16; k_new, v_new [B][Hkv][d] (or [B][Hkv][1][d]) bf16; the other
    arguments as for stief_decode_attention; max_seq_len bounds the lengths after the append.
    """
    pq = _dev(q, "q", torch.bfloat16, 3)
    kn = k_new.reshape(k_new.shape[0], k_new.shape[1], -1) if k_new.dim() == 4 else k_new
    vn = v_new.reshape(v_new.shape[0], v_new.shape[1], -1) if v_new.dim() == 4 else v_new
    pkn = _dev(kn, "k_new", torch.bfloat16, 3)
    pvn = _dev(vn, "v_new", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkl = _dev(k_lat, "k_lat", torch.bfloat16, 4)
    pvl = _dev(v_lat, "v_lat", torch.bfloat16, 4)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_V.shape[2]
    L_max = k_lat.shape[2]
    if tuple(P_K.shape) != (Hkv, d, rK) or tuple(P_V.shape) != (Hkv, d, rV) \
            or tuple(kn.shape) != (B, Hkv, d) or tuple(vn.shape) != (B, Hkv, d) \
            or tuple(k_lat.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_lat.shape) != (B, Hkv, L_max, rV) or seq_lens.shape[0] != B \
            or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_append_decode: inconsistent shapes")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_append_decode", (pq, pkn, pvn, ppk, ppv, pkl, pvl, psl, po,
                                         workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d, rK, rV,
                                         L_max, int(max_seq_len), int(num_splits),
                                         _opt_status(dev_status), _stream_ptr(stream),))
    return out


def _pages(k_pages, v_pages, block_table, B):
    """Pointers and sizes of a paged cache: pools [num_pages][Hkv][page_size][r] bf16 and a
    block table [B][max_pages] int32."""
    pkp = _dev(k_pages, "k_pages", torch.bfloat16, 4)
    pvp = _dev(v_pages, "v_pages", torch.bfloat16, 4)
    pbt = _dev(block_table, "block_table", torch.int32, 2)
    num_pages, Hkv, page_size, rK = k_pages.shape
    rV = v_pages.shape[3]
    if tuple(v_pages.shape) != (num_pages, Hkv, page_size, rV) or block_table.shape[0] != B:
        raise ValueError("paged cache: inconsistent shapes")
    return pkp, pvp, pbt, num_pages, Hkv, page_size, rK, rV, block_table.shape[1]


def stief_compress_append_paged(k_new, v_new, P_K, P_V, k_pages, v_pages, block_table, seq_lens,
                                dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """stief_compress_append into a paged cache (pools [num_pages][Hkv][page_size][r], block
    table [B][max_pages])."""
    pk = _dev(k_new, "k_new", torch.bfloat16, 4)
    pv = _dev(v_new, "v_new", torch.bfloat16, 4)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    B, Hkv, T, d = k_new.shape
    pkp, pvp, pbt, num_pages, Hkv2, page_size, rK, rV, max_pages = _pages(k_pages, v_pages,
                                                                          block_table, B)
    if Hkv2 != Hkv or tuple(P_K.shape) != (Hkv, d, rK) or tuple(P_V.shape) != (Hkv, d, rV) \
            or tuple(v_new.shape) != (B, Hkv, T, d) or seq_lens.shape[0] != B:
        raise ValueError("stief_compress_append_paged: inconsistent shapes")
    _invoke("stief_compress_append_paged", (pk, pv, ppk, ppv, pkp, pvp, pbt, psl, B, Hkv, T,
                                                 d, rK, rV, num_pages, page_size, max_pages,
                                                 _opt_status(dev_status), _stream_ptr(stream),))


def stief_decode_attention_paged(q, P_K, P_V, k_pages, v_pages, block_table, seq_lens, out,
                                 workspace, max_seq_len: int, num_splits: int = 0,
                                 dev_status: Optional[torch.Tensor] = None, stream=None):
    """stief_decode_attention over a paged cache."""
    pq = _dev(q, "q", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    B, Hq, d = q.shape
    pkp, pvp, pbt, num_pages, Hkv, page_size, rK, rV, max_pages = _pages(k_pages, v_pages,
                                                                         block_table, B)
    if tuple(P_K.shape) != (Hkv, d, rK) or tuple(P_V.shape) != (Hkv, d, rV) \
            or seq_lens.shape[0] != B or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_decode_attention_paged: inconsistent shapes")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_decode_attention_paged", (pq, ppk, ppv, pkp, pvp, pbt, psl, po,
                                                  workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d,
                                                  rK, rV, num_pages, page_size, max_pages,
                                                  int(max_seq_len), int(num_splits),
                                                  _opt_status(dev_status), _stream_ptr(stream),))
    return out


def stief_append_decode_paged(q, k_new, v_new, P_K, P_V, k_pages, v_pages, block_table, seq_lens,
                              out, workspace, max_seq_len: int, num_splits: int = 0,
                              dev_status: Optional[torch.Tensor] = None, stream=None):
    """stief_append_decode over a paged cache."""
    pq = _dev(q, "q", torch.bfloat16, 3)
    kn = k_new.reshape(k_new.shape[0], k_new.shape[1], -1) if k_new.dim() == 4 else k_new
    vn = v_new.reshape(v_new.shape[0], v_new.shape[1], -1) if v_new.dim() == 4 else v_new
    pkn = _dev(kn, "k_new", torch.bfloat16, 3)
    pvn = _dev(vn, "v_new", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    B, Hq, d = q.shape
    pkp, pvp, pbt, num_pages, Hkv, page_size, rK, rV, max_pages = _pages(k_pages, v_pages,
                                                                         block_table, B)
    if tuple(kn.shape) != (B, Hkv, d) or tuple(vn.shape) != (B, Hkv, d) \
            or tuple(P_K.shape) != (Hkv, d, rK) or tuple(P_V.shape) != (Hkv, d, rV) \
            or seq_lens.shape[0] != B or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_append_decode_paged: inconsistent shapes")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_append_decode_paged", (pq, pkn, pvn, ppk, ppv, pkp, pvp, pbt, psl, po,
                                               workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d, rK,
                                               rV, num_pages, page_size, max_pages,
                                               int(max_seq_len), int(num_splits),
                                               _opt_status(dev_status), _stream_ptr(stream),))
    return out


def stief_compress_append_q8(k_new, v_new, P_K, P_V, k_q, v_q, k_s, v_s, seq_lens,
                             dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """stief_compress_append into an int8 cache: codes k_q [B][Hkv][L_max][rK] (int8) and row
    scales k_s [B][Hkv][L_max] (float32), likewise v_q, v_s; L_max a multiple of 64."""
    pk = _dev(k_new, "k_new", torch.bfloat16, 4)
    pv = _dev(v_new, "v_new", torch.bfloat16, 4)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkq = _dev(k_q, "k_q", torch.int8, 4)
    pvq = _dev(v_q, "v_q", torch.int8, 4)
    pks = _dev(k_s, "k_s", torch.float32, 3)
    pvs = _dev(v_s, "v_s", torch.float32, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    B, Hkv, T, d = k_new.shape
    rK, rV = P_K.shape[2], P_V.shape[2]
    L_max = k_q.shape[2]
    if tuple(v_new.shape) != (B, Hkv, T, d) or tuple(P_K.shape) != (Hkv, d, rK) \
            or tuple(P_V.shape) != (Hkv, d, rV) or tuple(k_q.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_q.shape) != (B, Hkv, L_max, rV) or tuple(k_s.shape) != (B, Hkv, L_max) \
            or tuple(v_s.shape) != (B, Hkv, L_max) or seq_lens.shape[0] != B:
        raise ValueError("stief_compress_append_q8: inconsistent shapes")
    _invoke("stief_compress_append_q8", (pk, pv, ppk, ppv, pkq, pvq, pks, pvs, psl, B, Hkv, T,
                                              d, rK, rV, L_max, _opt_status(dev_status),
                                              _stream_ptr(stream),))


def stief_decode_attention_q8(q, P_K, P_V, k_q, v_q, k_s, v_s, seq_lens, out, workspace,
                              max_seq_len: int, num_splits: int = 0,
                              dev_status: Optional[torch.Tensor] = None, stream=None):
    """stief_decode_attention over an int8 cache (codes and row scales as for
    stief_compress_append_q8)."""
    pq = _dev(q, "q", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkq = _dev(k_q, "k_q", torch.int8, 4)
    pvq = _dev(v_q, "v_q", torch.int8, 4)
    pks = _dev(k_s, "k_s", torch.float32, 3)
    pvs = _dev(v_s, "v_s", torch.float32, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_V.shape[2]
    L_max = k_q.shape[2]
    if tuple(P_V.shape) != (Hkv, d, rV) or tuple(k_q.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_q.shape) != (B, Hkv, L_max, rV) or tuple(k_s.shape) != (B, Hkv, L_max) \
            or tuple(v_s.shape) != (B, Hkv, L_max) or seq_lens.shape[0] != B \
            or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_decode_attention_q8: inconsistent shapes")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_decode_attention_q8", (pq, ppk, ppv, pkq, pvq, pks, pvs, psl, po,
                                               workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d, rK,
                                               rV, L_max, int(max_seq_len), int(num_splits),
                                               _opt_status(dev_status), _stream_ptr(stream),))
    return out


def stief_append_decode_q8(q, k_new, v_new, P_K, P_V, k_q, v_q, k_s, v_s, seq_lens, out,
                           workspace, max_seq_len: int, num_splits: int = 0,
                           dev_status: Optional[torch.Tensor] = None, stream=None):
    """stief_append_decode on an int8 cache: the new token's rows are quantised into k_q, v_q
    (codes) and k_s, v_s (row scales) at row seq_lens[b] as stief_compress_append_q8 stores
    them, the decode attends over the grown cache, and seq_lens is incremented.  k_new, v_new
    [B][Hkv][d] (or [B][Hkv][1][d]) bf16; the rest as for stief_decode_attention_q8."""
    pq = _dev(q, "q", torch.bfloat16, 3)
    kn = k_new.reshape(k_new.shape[0], k_new.shape[1], -1) if k_new.dim() == 4 else k_new
    vn = v_new.reshape(v_new.shape[0], v_new.shape[1], -1) if v_new.dim() == 4 else v_new
    pkn = _dev(kn, "k_new", torch.bfloat16, 3)
    pvn = _dev(vn, "v_new", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkq = _dev(k_q, "k_q", torch.int8, 4)
    pvq = _dev(v_q, "v_q", torch.int8, 4)
    pks = _dev(k_s, "k_s", torch.float32, 3)
    pvs = _dev(v_s, "v_s", torch.float32, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_V.shape[2]
    L_max = k_q.shape[2]
    if tuple(P_V.shape) != (Hkv, d, rV) or tuple(kn.shape) != (B, Hkv, d) \
            or tuple(vn.shape) != (B, Hkv, d) or tuple(k_q.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_q.shape) != (B, Hkv, L_max, rV) or tuple(k_s.shape) != (B, Hkv, L_max) \
            or tuple(v_s.shape) != (B, Hkv, L_max) or seq_lens.shape[0] != B \
            or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_append_decode_q8: inconsistent shapes")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_append_decode_q8", (pq, pkn, pvn, ppk, ppv, pkq, pvq, pks, pvs, psl, po,
                                       workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d, rK, rV,
                                       L_max, int(max_seq_len), int(num_splits),
                                       _opt_status(dev_status), _stream_ptr(stream),))
    return out


def stief_compress_append_q8_paged(k_new, v_new, P_K, P_V, k_pages, v_pages, k_s_pages,
                                   v_s_pages, block_table, seq_lens,
                                   dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """stief_compress_append into int8 page pools: codes k_pages [num_pages][Hkv][page_size][rK]
    (int8) and row scales k_s_pages [num_pages][Hkv][page_size] (float32), likewise the values;
    block_table [B][max_pages] int32."""
    pk = _dev(k_new, "k_new", torch.bfloat16, 4)
    pv = _dev(v_new, "v_new", torch.bfloat16, 4)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkq = _dev(k_pages, "k_pages", torch.int8, 4)
    pvq = _dev(v_pages, "v_pages", torch.int8, 4)
    pks = _dev(k_s_pages, "k_s_pages", torch.float32, 3)
    pvs = _dev(v_s_pages, "v_s_pages", torch.float32, 3)
    pbt = _dev(block_table, "block_table", torch.int32, 2)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    B, Hkv, T, d = k_new.shape
    rK, rV = P_K.shape[2], P_V.shape[2]
    num_pages, _, page_size, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if tuple(v_new.shape) != (B, Hkv, T, d) or tuple(P_K.shape) != (Hkv, d, rK) \
            or tuple(P_V.shape) != (Hkv, d, rV) \
            or tuple(k_pages.shape) != (num_pages, Hkv, page_size, rK) \
            or tuple(v_pages.shape) != (num_pages, Hkv, page_size, rV) \
            or tuple(k_s_pages.shape) != (num_pages, Hkv, page_size) \
            or tuple(v_s_pages.shape) != (num_pages, Hkv, page_size) \
            or block_table.shape[0] != B or seq_lens.shape[0] != B:
        raise ValueError("stief_compress_append_q8_paged: inconsistent shapes")
    _invoke("stief_compress_append_q8_paged", (pk, pv, ppk, ppv, pkq, pvq, pks, pvs, pbt, psl,
                                                    B, Hkv, T, d, rK, rV, num_pages, page_size,
                                                    max_pages, _opt_status(dev_status),
                                                    _stream_ptr(stream),))


def stief_decode_attention_q8_paged(q, P_K, P_V, k_pages, v_pages, k_s_pages, v_s_pages,
                                    block_table, seq_lens, out, workspace, max_seq_len: int,
                                    num_splits: int = 0,
                                    dev_status: Optional[torch.Tensor] = None, stream=None):
    """stief_decode_attention over int8 page pools (as for stief_compress_append_q8_paged)."""
    pq = _dev(q, "q", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkq = _dev(k_pages, "k_pages", torch.int8, 4)
    pvq = _dev(v_pages, "v_pages", torch.int8, 4)
    pks = _dev(k_s_pages, "k_s_pages", torch.float32, 3)
    pvs = _dev(v_s_pages, "v_s_pages", torch.float32, 3)
    pbt = _dev(block_table, "block_table", torch.int32, 2)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_V.shape[2]
    num_pages, _, page_size, _ = k_pages.shape
    max_pages = block_table.shape[1]
    if tuple(P_V.shape) != (Hkv, d, rV) or tuple(k_pages.shape) != (num_pages, Hkv, page_size, rK) \
            or tuple(v_pages.shape) != (num_pages, Hkv, page_size, rV) \
            or tuple(k_s_pages.shape) != (num_pages, Hkv, page_size) \
            or tuple(v_s_pages.shape) != (num_pages, Hkv, page_size) \
            or block_table.shape[0] != B or seq_lens.shape[0] != B or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_decode_attention_q8_paged: inconsistent shapes")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_decode_attention_q8_paged", (pq, ppk, ppv, pkq, pvq, pks, pvs, pbt, psl, po,
                                                     workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d,
                                                     rK, rV, num_pages, page_size, max_pages,
                                                     int(max_seq_len), int(num_splits),
                                                     _opt_status(dev_status), _stream_ptr(stream),))
    return out


def stief_compress_append_q4(k_new, v_new, P_K, P_V, k_q, v_q, k_s, v_s, seq_lens,
                             dev_status: Optional[torch.Tensor] = None, stream=None) -> None:
    """stief_compress_append into a 4-bit cache: codes k_q [B][Hkv][L_max][rK / 2] (uint8, two
    per byte) and row scales k_s [B][Hkv][L_max] (float32), likewise v_q, v_s; ranks multiples
    of 32, L_max a multiple of 64."""
    pk = _dev(k_new, "k_new", torch.bfloat16, 4)
    pv = _dev(v_new, "v_new", torch.bfloat16, 4)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkq = _dev(k_q, "k_q", torch.uint8, 4)
    pvq = _dev(v_q, "v_q", torch.uint8, 4)
    pks = _dev(k_s, "k_s", torch.float32, 3)
    pvs = _dev(v_s, "v_s", torch.float32, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    B, Hkv, T, d = k_new.shape
    rK, rV = P_K.shape[2], P_V.shape[2]
    L_max = k_q.shape[2]
    if tuple(v_new.shape) != (B, Hkv, T, d) or tuple(P_K.shape) != (Hkv, d, rK) \
            or tuple(P_V.shape) != (Hkv, d, rV) or tuple(k_q.shape) != (B, Hkv, L_max, rK // 2) \
            or tuple(v_q.shape) != (B, Hkv, L_max, rV // 2) or tuple(k_s.shape) != (B, Hkv, L_max) \
            or tuple(v_s.shape) != (B, Hkv, L_max) or seq_lens.shape[0] != B:
        raise ValueError("stief_compress_append_q4: inconsistent shapes")
    _invoke("stief_compress_append_q4", (pk, pv, ppk, ppv, pkq, pvq, pks, pvs, psl, B, Hkv, T,
                                              d, rK, rV, L_max, _opt_status(dev_status),
                                              _stream_ptr(stream),))


def stief_decode_attention_q4(q, P_K, P_V, k_q, v_q, k_s, v_s, seq_lens, out, workspace,
                              max_seq_len: int, num_splits: int = 0,
                              dev_status: Optional[torch.Tensor] = None, stream=None):
    """stief_decode_attention over a 4-bit cache (codes and row scales as for
    stief_compress_append_q4)."""
    pq = _dev(q, "q", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkq = _dev(k_q, "k_q", torch.uint8, 4)
    pvq = _dev(v_q, "v_q", torch.uint8, 4)
    pks = _dev(k_s, "k_s", torch.float32, 3)
    pvs = _dev(v_s, "v_s", torch.float32, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_V.shape[2]
    L_max = k_q.shape[2]
    if tuple(P_V.shape) != (Hkv, d, rV) or tuple(k_q.shape) != (B, Hkv, L_max, rK // 2) \
            or tuple(v_q.shape) != (B, Hkv, L_max, rV // 2) or tuple(k_s.shape) != (B, Hkv, L_max) \
            or tuple(v_s.shape) != (B, Hkv, L_max) or seq_lens.shape[0] != B \
            or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_decode_attention_q4: inconsistent shapes")
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_decode_attention_q4", (pq, ppk, ppv, pkq, pvq, pks, pvs, psl, po,
                                               workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d, rK,
                                               rV, L_max, int(max_seq_len), int(num_splits),
                                               _opt_status(dev_status), _stream_ptr(stream),))
    return out


def stief_decode_latent(q_lat: torch.Tensor, k_lat: torch.Tensor, v_lat: torch.Tensor,
                        seq_lens: torch.Tensor, out_lat: torch.Tensor, workspace: torch.Tensor,
                        max_seq_len: int, num_splits: int = 0, d: int = 128,
                        dev_status: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The decode step in the latent space (bases folded into the attention weights):
    out_lat [B][Hq][rV] = softmax(q_lat k_lat^T / sqrt(d)) v_lat.

    q_lat [B][Hq][rK] bf16; k_lat [B][Hkv][L_max][rK], v_lat [B][Hkv][L_max][rV] bf16;
    seq_lens [B] int32; out_lat [B][Hq][rV] bf16 (written); d the head dimension (score
    scale); workspace as for stief_decode_attention.
    """
    pq = _dev(q_lat, "q_lat", torch.bfloat16, 3)
    pkl = _dev(k_lat, "k_lat", torch.bfloat16, 4)
    pvl = _dev(v_lat, "v_lat", torch.bfloat16, 4)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out_lat, "out_lat", torch.bfloat16, 3)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    B, Hq, rK = q_lat.shape
    Hkv, L_max = k_lat.shape[1], k_lat.shape[2]
    rV = v_lat.shape[3]
    if tuple(k_lat.shape) != (B, Hkv, L_max, rK) or tuple(v_lat.shape) != (B, Hkv, L_max, rV) \
            or seq_lens.shape[0] != B or tuple(out_lat.shape) != (B, Hq, rV):
        raise ValueError("stief_decode_latent: inconsistent shapes")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_decode_latent", (pq, pkl, pvl, psl, po, workspace.data_ptr(), ws_bytes,
                                         B, Hq, Hkv, int(d), rK, rV, L_max, int(max_seq_len),
                                         int(num_splits), _opt_status(dev_status),
                                         _stream_ptr(stream),))
    return out_lat


def stief_decode_attention_noalloc(q: torch.Tensor, P_K: torch.Tensor, P_V: torch.Tensor,
                                   k_lat: torch.Tensor, v_lat: torch.Tensor,
                                   seq_lens: torch.Tensor, out: torch.Tensor, max_seq_len: int,
                                   num_splits: int = 0, dev_status: Optional[torch.Tensor] = None,
                                   stream=None) -> torch.Tensor:
    """stief_decode_attention for callers that cannot allocate: no workspace argument.

    The library keeps the split partial states in its own fixed 8 MiB device array
    (one per GPU); calls that overlap on the GPU race on it.  Raises StiefError
    (STIEF_ERR_WORKSPACE) when the sizes need more than that.
    """
    pq = _dev(q, "q", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_V, "P_V", torch.bfloat16, 3)
    pkl = _dev(k_lat, "k_lat", torch.bfloat16, 4)
    pvl = _dev(v_lat, "v_lat", torch.bfloat16, 4)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_V.shape[2]
    L_max = k_lat.shape[2]
    if tuple(P_K.shape) != (Hkv, d, rK) or tuple(P_V.shape) != (Hkv, d, rV) \
            or tuple(k_lat.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_lat.shape) != (B, Hkv, L_max, rV) or seq_lens.shape[0] != B \
            or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_decode_attention_noalloc: inconsistent shapes")
    _invoke("stief_decode_attention_noalloc", (pq, ppk, ppv, pkl, pvl, psl, po, B, Hq, Hkv,
                                                    d, rK, rV, L_max, int(max_seq_len),
                                                    int(num_splits), _opt_status(dev_status),
                                                    _stream_ptr(stream),))
    return out


def stief_read_device_status(dev_status: torch.Tensor, stream=None) -> int:
    """Synchronise the stream and return the device status word (0 = no condition seen)."""
    v = ctypes.c_uint32(0)
    code = library().stief_read_device_status(_opt_status(dev_status), ctypes.byref(v),
                                              _stream_ptr(stream))
    if code not in (0, 6):
        raise StiefError("stief_read_device_status", code)
    return int(v.value)


def stief_decode_attention_joint_v(q: torch.Tensor, P_K: torch.Tensor, P_VJ: torch.Tensor,
                                   k_lat: torch.Tensor, v_joint: torch.Tensor,
                                   seq_lens: torch.Tensor, out: torch.Tensor,
                                   workspace: torch.Tensor, max_seq_len: int, num_splits: int = 0,
                                   dev_status: Optional[torch.Tensor] = None,
                                   stream=None) -> torch.Tensor:
    """stief_decode_attention with a joint value latent: P_VJ [Hkv*d][rV] bf16 over the
    concatenated KV-head values, v_joint [B][L_max][rV] bf16 (one row per token, shared by the
    KV heads); keys, q, out and the workspace as for stief_decode_attention."""
    pq = _dev(q, "q", torch.bfloat16, 3)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_VJ, "P_VJ", torch.bfloat16, 2)
    pkl = _dev(k_lat, "k_lat", torch.bfloat16, 4)
    pvl = _dev(v_joint, "v_joint", torch.bfloat16, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out, "out", torch.bfloat16, 3)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    B, Hq, d = q.shape
    Hkv, _, rK = P_K.shape
    rV = P_VJ.shape[1]
    L_max = k_lat.shape[2]
    if tuple(P_K.shape) != (Hkv, d, rK) or tuple(P_VJ.shape) != (Hkv * d, rV) \
            or tuple(k_lat.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_joint.shape) != (B, L_max, rV) or seq_lens.shape[0] != B \
            or tuple(out.shape) != (B, Hq, d):
        raise ValueError("stief_decode_attention_joint_v: inconsistent shapes")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_decode_attention_joint_v", (pq, ppk, ppv, pkl, pvl, psl, po,
                                                    workspace.data_ptr(), ws_bytes, B, Hq, Hkv, d,
                                                    rK, rV, L_max, int(max_seq_len),
                                                    int(num_splits), _opt_status(dev_status),
                                                    _stream_ptr(stream),))
    return out


def stief_decode_latent_joint_v(q_lat: torch.Tensor, k_lat: torch.Tensor, v_joint: torch.Tensor,
                                seq_lens: torch.Tensor, out_lat: torch.Tensor,
                                workspace: torch.Tensor, max_seq_len: int, num_splits: int = 0,
                                d: int = 128, dev_status: Optional[torch.Tensor] = None,
                                stream=None) -> torch.Tensor:
    """stief_decode_latent with a joint value latent v_joint [B][L_max][rV] bf16 (one row per
    token, shared by the KV heads)."""
    pq = _dev(q_lat, "q_lat", torch.bfloat16, 3)
    pkl = _dev(k_lat, "k_lat", torch.bfloat16, 4)
    pvl = _dev(v_joint, "v_joint", torch.bfloat16, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    po = _dev(out_lat, "out_lat", torch.bfloat16, 3)
    if not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous CUDA tensor")
    B, Hq, rK = q_lat.shape
    Hkv, L_max = k_lat.shape[1], k_lat.shape[2]
    rV = v_joint.shape[2]
    if tuple(k_lat.shape) != (B, Hkv, L_max, rK) or tuple(v_joint.shape) != (B, L_max, rV) \
            or seq_lens.shape[0] != B or tuple(out_lat.shape) != (B, Hq, rV):
        raise ValueError("stief_decode_latent_joint_v: inconsistent shapes")
    ws_bytes = workspace.numel() * workspace.element_size()
    _invoke("stief_decode_latent_joint_v", (pq, pkl, pvl, psl, po, workspace.data_ptr(),
                                                 ws_bytes, B, Hq, Hkv, int(d), rK, rV, L_max,
                                                 int(max_seq_len), int(num_splits),
                                                 _opt_status(dev_status), _stream_ptr(stream),))
    return out_lat


def stief_compress_append_joint_v(k_new: torch.Tensor, v_new: torch.Tensor, P_K: torch.Tensor,
                                  P_VJ: torch.Tensor, k_lat: torch.Tensor, v_joint: torch.Tensor,
                                  seq_lens: torch.Tensor, dev_status: Optional[torch.Tensor] = None,
                                  stream=None) -> None:
    """stief_compress_append with the values projected jointly over the KV heads: keys per head
    into k_lat [B][Hkv][L_max][rK], values through P_VJ [Hkv*d][rV] into v_joint [B][L_max][rV]
    (one row per token); k_new, v_new [B][Hkv][T][d] bf16; seq_lens [B] int32 advanced by T."""
    pk = _dev(k_new, "k_new", torch.bfloat16, 4)
    pv = _dev(v_new, "v_new", torch.bfloat16, 4)
    ppk = _dev(P_K, "P_K", torch.bfloat16, 3)
    ppv = _dev(P_VJ, "P_VJ", torch.bfloat16, 2)
    pkl = _dev(k_lat, "k_lat", torch.bfloat16, 4)
    pvl = _dev(v_joint, "v_joint", torch.bfloat16, 3)
    psl = _dev(seq_lens, "seq_lens", torch.int32, 1)
    B, Hkv, T, d = k_new.shape
    rK, rV = P_K.shape[2], P_VJ.shape[1]
    L_max = k_lat.shape[2]
    if tuple(v_new.shape) != (B, Hkv, T, d) or tuple(P_K.shape) != (Hkv, d, rK) \
            or tuple(P_VJ.shape) != (Hkv * d, rV) or tuple(k_lat.shape) != (B, Hkv, L_max, rK) \
            or tuple(v_joint.shape) != (B, L_max, rV) or seq_lens.shape[0] != B:
        raise ValueError("stief_compress_append_joint_v: inconsistent shapes")
    _invoke("stief_compress_append_joint_v", (pk, pv, ppk, ppv, pkl, pvl, psl, B, Hkv, T, d,
                                                   rK, rV, L_max, _opt_status(dev_status),
                                                   _stream_ptr(stream),))
