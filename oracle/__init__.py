"""Plain fp64 CPU oracle for StiefAttention latent-KV decode (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm
of ``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it and has no CPU fallback.

The arithmetic lives in ``stief_oracle.c`` (plain C, IEEE double, sequential sums
in the order of the definition).  This module only converts numpy arrays to
contiguous float64 / int32 buffers and calls it through ctypes.  The C source is
compiled with gcc on first use if the shared object is missing or stale; no
flags that reorder floating point (no -ffast-math) are used.

Definitions followed (StiefAttention technical summary, "Mecanismo Central" /
"Kernmechanismus", items 2 and 5): stored latent ``K_down = K . P_K`` and
``V_down = V . P_V``; on-the-fly reconstruction ``K~ = K_down . P_K^T`` and
``V~ = V_down . P_V^T`` before softmax attention.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "stief_oracle.c")
_LIB = os.path.join(_HERE, "libstief_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I32 = ctypes.POINTER(ctypes.c_int32)


def build(src: str = _SRC, out: str = _LIB, force: bool = False) -> str:
    """Compile the oracle C source into a shared object (gcc -O2, OpenMP, no fast-math)."""
    stale = (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)
    if force or stale:
        tmp = out + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
               "-fno-fast-math", "-ffp-contract=off", src, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray, typ=_D):
    return a.ctypes.data_as(typ)


class Oracle:
    """ctypes view of one compiled oracle shared object."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.stief_oracle_round_bf16.restype = ctypes.c_double
        lib.stief_oracle_round_bf16.argtypes = [ctypes.c_double]
        lib.stief_oracle_round_bf16_array.restype = None
        lib.stief_oracle_round_bf16_array.argtypes = [_D, _D, ctypes.c_long]
        lib.stief_oracle_project.restype = None
        lib.stief_oracle_project.argtypes = [_D, _D, _D, ctypes.c_long, ctypes.c_int,
                                             ctypes.c_int, ctypes.c_int]
        lib.stief_oracle_compress_append.restype = ctypes.c_int
        lib.stief_oracle_compress_append.argtypes = (
            [_D, _D, _D, _D, _D, _D, _I32] + [ctypes.c_int] * 8)
        lib.stief_oracle_decode.restype = ctypes.c_int
        lib.stief_oracle_decode.argtypes = (
            [_D, _D, _D, _D, _D, _I32, _D] + [ctypes.c_int] * 8)
        lib.stief_oracle_decode_latent.restype = ctypes.c_int
        lib.stief_oracle_decode_latent.argtypes = (
            [_D, _D, _D, _I32, _D] + [ctypes.c_int] * 8)
        lib.stief_oracle_max_threads.restype = ctypes.c_int
        lib.stief_oracle_max_threads.argtypes = []
        self.lib = lib
        self.path = path

    def max_threads(self) -> int:
        """OpenMP threads a decode call uses by default."""
        return int(self.lib.stief_oracle_max_threads())

    def round_bf16(self, x) -> np.ndarray:
        """Round every element to the nearest bfloat16 value, ties to even (fp64 result)."""
        x = _f64(x)
        y = np.empty_like(x)
        self.lib.stief_oracle_round_bf16_array(_ptr(x), _ptr(y), x.size)
        return y

    def project(self, x, P, round_to_bf16: bool = True) -> np.ndarray:
        """Compressed storage of rows: y = x . P (x [T][d], P [d][r]), optionally bf16-rounded."""
        x = _f64(x)
        P = _f64(P)
        T, d = x.shape
        d2, r = P.shape
        if d2 != d:
            raise ValueError("project: inner dimensions differ")
        y = np.empty((T, r), dtype=np.float64)
        self.lib.stief_oracle_project(_ptr(x), _ptr(P), _ptr(y), T, d, r, int(round_to_bf16))
        return y

    def compress_append(self, k_new, v_new, P_K, P_V, k_lat, v_lat, seq_lens,
                        round_to_bf16: bool = True):
        """Append T projected rows per (sequence, KV head).

        Shapes: k_new/v_new [B][Hkv][T][d], P_K [Hkv][d][rK], P_V [Hkv][d][rV],
        k_lat [B][Hkv][L_max][rK], v_lat [B][Hkv][L_max][rV], seq_lens [B].
        The inputs are not modified; returns (k_lat, v_lat, seq_lens, n_overflow)
        as updated copies.
        """
        k_new, v_new, P_K, P_V = map(_f64, (k_new, v_new, P_K, P_V))
        k_lat = _f64(k_lat).copy()
        v_lat = _f64(v_lat).copy()
        lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32)).copy()
        B, Hkv, T, d = k_new.shape
        rK = P_K.shape[2]
        rV = P_V.shape[2]
        L_max = k_lat.shape[2]
        if v_new.shape != k_new.shape or P_K.shape[:2] != (Hkv, d) or P_V.shape[:2] != (Hkv, d):
            raise ValueError("compress_append: inconsistent shapes")
        if k_lat.shape != (B, Hkv, L_max, rK) or v_lat.shape != (B, Hkv, L_max, rV):
            raise ValueError("compress_append: inconsistent cache shapes")
        n_bad = self.lib.stief_oracle_compress_append(
            _ptr(k_new), _ptr(v_new), _ptr(P_K), _ptr(P_V), _ptr(k_lat), _ptr(v_lat),
            _ptr(lens, _I32), B, Hkv, T, d, rK, rV, L_max, int(round_to_bf16))
        return k_lat, v_lat, lens, int(n_bad)

    def decode(self, q, P_K, P_V, k_lat, v_lat, seq_lens, num_threads: int = 0) -> np.ndarray:
        """One decode step over the reconstructed latent cache; returns out [B][Hq][d] (fp64).

        Shapes: q [B][Hq][d], P_K [Hkv][d][rK], P_V [Hkv][d][rV],
        k_lat [B][Hkv][L_max][rK], v_lat [B][Hkv][L_max][rV], seq_lens [B].
        """
        q, P_K, P_V, k_lat, v_lat = map(_f64, (q, P_K, P_V, k_lat, v_lat))
        lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
        B, Hq, d = q.shape
        Hkv, d2, rK = P_K.shape
        rV = P_V.shape[2]
        L_max = k_lat.shape[2]
        if d2 != d or Hq % Hkv != 0 or P_V.shape[:2] != (Hkv, d):
            raise ValueError("decode: inconsistent shapes")
        if k_lat.shape != (B, Hkv, L_max, rK) or v_lat.shape != (B, Hkv, L_max, rV):
            raise ValueError("decode: inconsistent cache shapes")
        out = np.empty((B, Hq, d), dtype=np.float64)
        rc = self.lib.stief_oracle_decode(_ptr(q), _ptr(P_K), _ptr(P_V), _ptr(k_lat),
                                          _ptr(v_lat), _ptr(lens, _I32), _ptr(out),
                                          B, Hq, Hkv, d, rK, rV, L_max, int(num_threads))
        if rc != 0:
            raise ValueError("decode: a sequence length is outside [0, L_max]")
        return out


    def decode_latent(self, q_lat, k_lat, v_lat, seq_lens, d: int = 128,
                      num_threads: int = 0) -> np.ndarray:
        """Decode in the latent space (bases folded into the attention weights); returns
        o~ [B][Hq][rV] (fp64).  Scores are scaled by 1/sqrt(d), d the full head dimension.

        Shapes: q_lat [B][Hq][rK], k_lat [B][Hkv][L_max][rK], v_lat [B][Hkv][L_max][rV],
        seq_lens [B].
        """
        q_lat, k_lat, v_lat = map(_f64, (q_lat, k_lat, v_lat))
        lens = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
        B, Hq, rK = q_lat.shape
        Hkv, L_max = k_lat.shape[1], k_lat.shape[2]
        rV = v_lat.shape[3]
        if Hq % Hkv != 0 or k_lat.shape != (B, Hkv, L_max, rK) \
                or v_lat.shape != (B, Hkv, L_max, rV):
            raise ValueError("decode_latent: inconsistent shapes")
        out = np.empty((B, Hq, rV), dtype=np.float64)
        rc = self.lib.stief_oracle_decode_latent(_ptr(q_lat), _ptr(k_lat), _ptr(v_lat),
                                                 _ptr(lens, _I32), _ptr(out), B, Hq, Hkv, int(d),
                                                 rK, rV, L_max, int(num_threads))
        if rc != 0:
            raise ValueError("decode_latent: a sequence length is outside [0, L_max]")
        return out

    # ------------------------------------------------------------------ joint value latent
    #
    # STAR-KV technical summary, "Metodologia" item 2 (hybrid decomposition): the keys keep
    # one basis per KV head, the values of all KV heads are factored together.  The joint
    # value basis P_VJ is [Hkv*d][rV] over the concatenation v_cat = [v_0 | v_1 | ... ] of a
    # token's KV-head value rows, and the cache stores one value latent per token,
    # v_joint = v_cat . P_VJ, shared by every head.  Reconstruction gives the whole
    # concatenation back, v_cat~ = v_joint . P_VJ^T, and KV head g reads its own block of d
    # coordinates, [g*d, (g+1)*d).  The three helpers below are that layout and nothing else;
    # every product runs in the C functions above.

    @staticmethod
    def _concat_heads(x):
        """[Hkv][T][d] -> [T][Hkv*d]: a token's KV-head rows side by side, head 0 first."""
        Hkv, T, d = x.shape
        return np.ascontiguousarray(np.transpose(x, (1, 0, 2)).reshape(T, Hkv * d))

    @staticmethod
    def _head_blocks(P_VJ, Hkv):
        """[Hkv*d][rV] -> [Hkv][d][rV]: block g holds rows [g*d, (g+1)*d) of P_VJ, the part of
        the reconstruction that lands in KV head g's coordinates."""
        HD, rV = P_VJ.shape
        return np.ascontiguousarray(P_VJ.reshape(Hkv, HD // Hkv, rV))

    @staticmethod
    def _share_values(v_joint, Hkv):
        """[B][L][rV] -> [B][Hkv][L][rV]: the one value latent of a token, seen by each head."""
        B, L, rV = v_joint.shape
        return np.ascontiguousarray(np.broadcast_to(v_joint[:, None], (B, Hkv, L, rV)))

    def compress_append_joint_v(self, k_new, v_new, P_K, P_VJ, k_lat, v_joint, seq_lens,
                                round_to_bf16: bool = True):
        """Append T tokens per sequence: keys per KV head (k_lat[b][g] gets k_new[b][g] . P_K[g]),
        values jointly (v_joint[b] gets concat_g(v_new[b][g]) . P_VJ), both bf16-rounded like
        the per-head cache.  A sequence whose rows would pass L_max is left untouched and
        counted.

        Shapes: k_new/v_new [B][Hkv][T][d], P_K [Hkv][d][rK], P_VJ [Hkv*d][rV],
        k_lat [B][Hkv][L_max][rK], v_joint [B][L_max][rV], seq_lens [B].
        Returns updated copies (k_lat, v_joint, seq_lens, n_overflow).
        """
        k_new, v_new, P_K, P_VJ = map(_f64, (k_new, v_new, P_K, P_VJ))
        k_lat = _f64(k_lat).copy()
        v_joint = _f64(v_joint).copy()
        lens = np.asarray(seq_lens, dtype=np.int32).copy()
        B, Hkv, T, d = k_new.shape
        L_max = k_lat.shape[2]
        if v_new.shape != k_new.shape or P_K.shape[:2] != (Hkv, d) or P_VJ.shape[0] != Hkv * d:
            raise ValueError("compress_append_joint_v: inconsistent shapes")
        if k_lat.shape[:2] != (B, Hkv) or v_joint.shape[:2] != (B, L_max):
            raise ValueError("compress_append_joint_v: inconsistent cache shapes")
        n_bad = 0
        for b in range(B):
            L = int(lens[b])
            if L < 0 or L + T > L_max:
                n_bad += 1
                continue
            for g in range(Hkv):
                k_lat[b, g, L:L + T] = self.project(k_new[b, g], P_K[g], round_to_bf16)
            v_joint[b, L:L + T] = self.project(self._concat_heads(v_new[b]), P_VJ, round_to_bf16)
            lens[b] = L + T
        return k_lat, v_joint, lens, n_bad

    def decode_joint_v(self, q, P_K, P_VJ, k_lat, v_joint, seq_lens,
                       num_threads: int = 0) -> np.ndarray:
        """One decode step with per-head keys and a joint value latent; returns [B][Hq][d].

        Query head h of KV head g: scores against K_down[g] . P_K[g]^T as in decode(); its
        values are block g of v_joint[t] . P_VJ^T.  That is decode() with P_V[g] = block g of
        P_VJ and every head reading the shared value latent.
        Shapes: q [B][Hq][d], P_K [Hkv][d][rK], P_VJ [Hkv*d][rV], k_lat [B][Hkv][L_max][rK],
        v_joint [B][L_max][rV], seq_lens [B].
        """
        P_K, P_VJ, v_joint = map(_f64, (P_K, P_VJ, v_joint))
        Hkv = P_K.shape[0]
        if P_VJ.shape[0] != Hkv * P_K.shape[1] or v_joint.ndim != 3:
            raise ValueError("decode_joint_v: inconsistent shapes")
        return self.decode(q, P_K, self._head_blocks(P_VJ, Hkv), k_lat,
                           self._share_values(v_joint, Hkv), seq_lens, num_threads)

    def decode_latent_joint_v(self, q_lat, k_lat, v_joint, seq_lens, d: int = 128,
                              num_threads: int = 0) -> np.ndarray:
        """Latent-space decode with a joint value latent (bases folded into the weights; the
        output projection absorbs block g of P_VJ); returns o~ [B][Hq][rV].

        Shapes: q_lat [B][Hq][rK], k_lat [B][Hkv][L_max][rK], v_joint [B][L_max][rV].
        """
        k_lat, v_joint = _f64(k_lat), _f64(v_joint)
        return self.decode_latent(q_lat, k_lat, self._share_values(v_joint, k_lat.shape[1]),
                                  seq_lens, d, num_threads)

def default() -> Oracle:
    """The oracle built from stief_oracle.c (compiled on first use)."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle(build())
    return _lib


def max_threads() -> int:
    return default().max_threads()


def round_bf16(x) -> np.ndarray:
    return default().round_bf16(x)


def project(x, P, round_to_bf16: bool = True) -> np.ndarray:
    return default().project(x, P, round_to_bf16)


def compress_append(k_new, v_new, P_K, P_V, k_lat, v_lat, seq_lens, round_to_bf16: bool = True):
    return default().compress_append(k_new, v_new, P_K, P_V, k_lat, v_lat, seq_lens,
                                     round_to_bf16)


def decode(q, P_K, P_V, k_lat, v_lat, seq_lens, num_threads: int = 0) -> np.ndarray:
    return default().decode(q, P_K, P_V, k_lat, v_lat, seq_lens, num_threads)


def decode_latent(q_lat, k_lat, v_lat, seq_lens, d: int = 128, num_threads: int = 0) -> np.ndarray:
    return default().decode_latent(q_lat, k_lat, v_lat, seq_lens, d, num_threads)


def gather_pages(pages, block_table, seq_lens, L_max: int) -> np.ndarray:
    """The contiguous cache [B][Hkv][L_max][r] (fp64) that a paged cache stands for.

    The library's paged layout: a pool ``pages`` [num_pages][Hkv][page_size][r] and a block
    table [B][max_pages]; token t of (sequence b, KV head h) is row t % page_size of page
    block_table[b][t // page_size], head h.  Rows at and past seq_lens[b] are left zero.
    Plain indexing, no arithmetic: the paged calls are defined as the contiguous ones on the
    cache this returns.
    """
    pages = _f64(pages)
    bt = np.asarray(block_table)
    lens = np.asarray(seq_lens)
    num_pages, Hkv, ps, r = pages.shape
    B = bt.shape[0]
    out = np.zeros((B, Hkv, L_max, r), dtype=np.float64)
    for b in range(B):
        for t in range(int(lens[b])):
            out[b, :, t] = pages[int(bt[b, t // ps]), :, t % ps]
    return out


def quantize_rows(x, qmax: int = 127):
    """Per-row symmetric quantisation of latent rows (the low-bit cache forms).

    The pages report the compressed cache to be robust to 4- and 8-bit quantisation but fix no
    scheme; this library's reading: one fp32 scale per stored row (per token, KV head),
        scale = fp32(max_c |x_c| / qmax),  code_c = RNE(fp32(x_c / scale)) in [-qmax, qmax],
    qmax = 127 for the int8 form and 7 for the 4-bit form, with a zero row stored as scale 0
    and codes 0.  x are the bf16 latent values (exact in fp32).  The two divisions and the
    rounding to an integer are taken in IEEE fp32, the kernel's precision, so the integer codes
    are decided identically on both sides.
    Returns (codes int8 [..., r], scales float32 [...]).
    """
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    scale = (amax / np.float32(qmax)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    q = np.rint((x32 / safe[..., None]).astype(np.float32))
    q = np.where(scale[..., None] > 0, q, 0.0)
    return np.clip(q, -qmax, qmax).astype(np.int8), scale


def pack_q4(codes) -> np.ndarray:
    """4-bit codes in [-8, 7] (int8 [..., r], r even) two per byte: byte j holds column 2j in
    its low nibble and column 2j + 1 in its high nibble, each as a 4-bit two's complement."""
    c = np.asarray(codes, dtype=np.int16)
    lo = c[..., 0::2] & 0xF
    hi = c[..., 1::2] & 0xF
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_q4(packed) -> np.ndarray:
    """The inverse of pack_q4: uint8 [..., r / 2] -> int8 codes [..., r]."""
    p = np.asarray(packed, dtype=np.int16)
    lo = p & 0xF
    hi = (p >> 4) & 0xF
    lo = np.where(lo >= 8, lo - 16, lo)
    hi = np.where(hi >= 8, hi - 16, hi)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.int8)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return out


def dequantize_rows(codes, scales) -> np.ndarray:
    """code * scale per element, exact in fp64."""
    return np.asarray(codes, np.float64) * np.asarray(scales, np.float64)[..., None]



def compress_append_joint_v(k_new, v_new, P_K, P_VJ, k_lat, v_joint, seq_lens,
                            round_to_bf16: bool = True):
    return default().compress_append_joint_v(k_new, v_new, P_K, P_VJ, k_lat, v_joint, seq_lens,
                                             round_to_bf16)


def decode_joint_v(q, P_K, P_VJ, k_lat, v_joint, seq_lens, num_threads: int = 0) -> np.ndarray:
    return default().decode_joint_v(q, P_K, P_VJ, k_lat, v_joint, seq_lens, num_threads)


def decode_latent_joint_v(q_lat, k_lat, v_joint, seq_lens, d: int = 128,
                          num_threads: int = 0) -> np.ndarray:
    return default().decode_latent_joint_v(q_lat, k_lat, v_joint, seq_lens, d, num_threads)
