"""CPU fp64 oracle for the R-SWA / SR-SWA decode-attention hot path.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package. The product path (``long_context_decode_swa_b200``) never imports it
and shares no code with it.

The arithmetic lives in ``rswa_oracle.c`` (plain C, fp64, OpenMP over
independent (sequence, head) problems); this module compiles it with gcc on
first use and marshals numpy arrays. bf16 tensors travel as their raw 16-bit
patterns in ``np.uint16`` arrays. ``kv_cache_bytes`` is the one piece of
arithmetic written here, in Python: the cache-size closed form.

Parity status: every function is pinned by ``tests/test_oracle_*.py`` (see
each function's docstring for its pins); none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rswa_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 32  # SR-SWA block size (sparse_block_size)


def build(force: bool = False) -> str:
    """Compile the oracle library with gcc (no GPU involved). Returns its path."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _L():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            I64 = ctypes.c_int64
            Dbl = ctypes.c_double
            lib.oracle_set_threads.argtypes = [I]
            lib.oracle_get_threads.restype = I
            lib.oracle_append.argtypes = [I, I, I, I, P, P, P, P, P, P, P]
            lib.oracle_rswa_decode.argtypes = [I, I, I, I, I64, P, P, P, P, P, P, P, P, Dbl, P, P]
            lib.oracle_rswa_prefill.argtypes = [I, I, I, I, I64, I, P, P, P, P, P, P, P, P, P, P, Dbl, P, I, P, P]
            lib.oracle_index_pool.argtypes = [I, I64, I, I, P, P, P]
            lib.oracle_entmax15.argtypes = [I64, P, P]
            lib.oracle_entmax15.restype = Dbl
            lib.oracle_route.argtypes = [I, I64, I, I, P, P, P, Dbl, I, P, P, P, P, P]
            lib.oracle_srswa_decode.argtypes = [I, I, I, I, I64, I, P, P, P, P, P, P, I, P, P, P, P, Dbl, P, P]
            lib.oracle_route_tokens.argtypes = [I, I, I64, I, I, P, P, P, Dbl, I, P, P]
            lib.oracle_srswa_prefill.argtypes = [I, I, I, I, I64, I, I, P, P, P, P, P, P, P, P, I, P, P, P, P, Dbl,
                                                 P, I, P, P]
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_to_double.restype = Dbl
            lib.oracle_e4m3_encode.argtypes = [ctypes.c_float]
            lib.oracle_e4m3_encode.restype = ctypes.c_uint8
            lib.oracle_e4m3_encode_array.argtypes = [I64, P, P]
            lib.oracle_quantize_prefix.argtypes = [I, I, I, I64, I, P, P, P, P]
            lib.oracle_rswa_decode_fp8.argtypes = [I, I, I, I, I64, I, P, P, P, P, P, P, P, P, P, P, Dbl, P, P]
            lib.oracle_srswa_decode_fp8.argtypes = [I, I, I, I, I64, I, P, P, P, P, P, P, P, P, I, P, P, P, P, Dbl,
                                                    P, P]
            lib.oracle_bf16_round.argtypes = [Dbl]
            lib.oracle_bf16_round.restype = ctypes.c_uint16
            lib.oracle_bf16_round_array.argtypes = [I64, P, P]
            lib.oracle_rope_page2d.argtypes = [I64, I, I, P, P, P, Dbl, I, P]
            lib.oracle_append_fp8.argtypes = [I, I, I, I, P, P, P, P, P, P, P, P, P]
            lib.oracle_rswa_decode_fp8kv.argtypes = [I, I, I, I, I64, I, P, P, P, P, P, P, P, P, P, P, P, P, Dbl,
                                                     P, P]
            lib.oracle_srswa_decode_fp8kv.argtypes = [I, I, I, I, I64, I, P, P, P, P, P, P, P, P, I, P, P, P, P, P,
                                                      P, Dbl, P, P]
            _lib = lib
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a, ndim: int, name: str) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"{name}: expected bf16 bit patterns as uint16, got {a.dtype}")
    if a.ndim != ndim:
        raise ValueError(f"{name}: expected {ndim} dims, got shape {a.shape}")
    return a


def _i32(a, name: str) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.int32:
        raise TypeError(f"{name}: expected int32, got {a.dtype}")
    return a


def set_threads(n: int) -> None:
    _L().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_L().oracle_get_threads())


def append(ring_k, ring_v, k_new, v_new, wp, fill):
    """Ring append, in place on ring_k/ring_v/wp/fill. Returns slot_out [B].

    ring_* uint16 [B][H][n][D]; k_new/v_new uint16 [B][H][D]; wp/fill int32 [B].
    """
    for name, a in (("ring_k", ring_k), ("ring_v", ring_v), ("wp", wp), ("fill", fill)):
        if not (isinstance(a, np.ndarray) and a.flags.c_contiguous):
            raise ValueError(f"{name} must be a C-contiguous numpy array (updated in place)")
    B, H, n, D = ring_k.shape
    k_new = _u16(k_new, 3, "k_new")
    v_new = _u16(v_new, 3, "v_new")
    slot = np.zeros(B, np.int32)
    _L().oracle_append(B, H, n, D, _p(ring_k), _p(ring_v), _p(k_new), _p(v_new), _p(wp), _p(fill), _p(slot))
    return slot


def rswa_decode(q, pk, pv, prefix_len, ring_k, ring_v, wp, fill, scale):
    """R-SWA decode for every (b, h). Returns (out fp64 [B][H][D], lse fp64 [B][H])."""
    q = _u16(q, 3, "q")
    pk = _u16(pk, 4, "pk")
    pv = _u16(pv, 4, "pv")
    ring_k = _u16(ring_k, 4, "ring_k")
    ring_v = _u16(ring_v, 4, "ring_v")
    prefix_len, wp, fill = _i32(prefix_len, "prefix_len"), _i32(wp, "wp"), _i32(fill, "fill")
    B, H, D = q.shape
    cap = pk.shape[2]
    n = ring_k.shape[2]
    out = np.zeros((B, H, D), np.float64)
    lse = np.zeros((B, H), np.float64)
    _L().oracle_rswa_decode(B, H, D, n, cap, _p(q), _p(pk), _p(pv), _p(prefix_len), _p(ring_k), _p(ring_v),
                            _p(wp), _p(fill), float(scale), _p(out), _p(lse))
    return out, lse


def rswa_prefill(q, k_out, v_out, pk, pv, prefix_len, scale, rows, n, ring_k=None, ring_v=None, wp=None, fill=None):
    """R-SWA prefill for the listed query rows. Returns (out [B][H][R][D], lse [B][H][R]).

    q/k_out/v_out uint16 [B][H][T][D]; ring (optional) holds the previous chunk.
    """
    q = _u16(q, 4, "q")
    k_out = _u16(k_out, 4, "k_out")
    v_out = _u16(v_out, 4, "v_out")
    pk = _u16(pk, 4, "pk")
    pv = _u16(pv, 4, "pv")
    B, H, T, D = q.shape
    cap = pk.shape[2]
    prefix_len = _i32(prefix_len, "prefix_len")
    rows = _i32(np.asarray(rows, np.int32), "rows")
    if rows.size and (rows.min() < 0 or rows.max() >= T):
        raise ValueError("row index out of range")
    if ring_k is not None:
        ring_k = _u16(ring_k, 4, "ring_k")
        ring_v = _u16(ring_v, 4, "ring_v")
        wp, fill = _i32(wp, "wp"), _i32(fill, "fill")
        if ring_k.shape[2] != n:
            raise ValueError("ring slots != n")
    R = rows.size
    out = np.zeros((B, H, R, D), np.float64)
    lse = np.zeros((B, H, R), np.float64)
    _L().oracle_rswa_prefill(B, H, D, int(n), cap, T, _p(q), _p(k_out), _p(v_out), _p(pk), _p(pv), _p(prefix_len),
                             _p(ring_k), _p(ring_v), _p(wp), _p(fill), float(scale), _p(rows), R, _p(out), _p(lse))
    return out, lse


def index_pool(k_idx, prefix_len, blk: int = BLOCK):
    """Block index keys: kbar fp64 [B][ceil(cap/blk)][DI] (mean of valid token keys)."""
    k_idx = _u16(k_idx, 3, "k_idx")
    prefix_len = _i32(prefix_len, "prefix_len")
    B, cap, DI = k_idx.shape
    nb_cap = (cap + blk - 1) // blk
    kbar = np.zeros((B, nb_cap, DI), np.float64)
    _L().oracle_index_pool(B, cap, DI, blk, _p(k_idx), _p(prefix_len), _p(kbar))
    return kbar


def entmax15(x):
    """Exact 1.5-entmax of x (x already = z/2). Returns (p fp64, tau)."""
    x = np.ascontiguousarray(np.asarray(x, np.float64).ravel())
    p = np.zeros_like(x)
    tau = _L().oracle_entmax15(x.size, _p(x), _p(p))
    return p, float(tau)


def route(q_idx, kbar, prefix_len, topk: int = 16, idx_scale: float = 1.0, blk: int = BLOCK):
    """Router: returns dict(blk_idx int32 [B][topk], blk_logp fp64, probs fp64 [B][NBcap], tau fp64 [B], z fp64)."""
    q_idx = np.ascontiguousarray(q_idx, np.float32)
    kbar = np.ascontiguousarray(kbar, np.float64)
    prefix_len = _i32(prefix_len, "prefix_len")
    B, nb_cap, DI = kbar.shape
    if q_idx.shape != (B, DI):
        raise ValueError("q_idx shape")
    blk_idx = np.zeros((B, topk), np.int32)
    blk_logp = np.zeros((B, topk), np.float64)
    probs = np.zeros((B, nb_cap), np.float64)
    tau = np.zeros(B, np.float64)
    z = np.zeros((B, nb_cap), np.float64)
    _L().oracle_route(B, nb_cap, DI, blk, _p(q_idx), _p(kbar), _p(prefix_len), float(idx_scale), int(topk),
                      _p(blk_idx), _p(blk_logp), _p(probs), _p(tau), _p(z))
    return dict(blk_idx=blk_idx, blk_logp=blk_logp, probs=probs, tau=tau, z=z)


def srswa_decode(q, pk, pv, prefix_len, blk_idx, blk_logp, ring_k, ring_v, wp, fill, scale, blk: int = BLOCK):
    """SR-SWA gathered-block decode. Returns (out fp64 [B][H][D], lse fp64 [B][H])."""
    q = _u16(q, 3, "q")
    pk = _u16(pk, 4, "pk")
    pv = _u16(pv, 4, "pv")
    ring_k = _u16(ring_k, 4, "ring_k")
    ring_v = _u16(ring_v, 4, "ring_v")
    prefix_len, wp, fill = _i32(prefix_len, "prefix_len"), _i32(wp, "wp"), _i32(fill, "fill")
    blk_idx = _i32(blk_idx, "blk_idx")
    blk_logp = np.ascontiguousarray(blk_logp, np.float64)
    B, H, D = q.shape
    topk = blk_idx.shape[1]
    cap = pk.shape[2]
    n = ring_k.shape[2]
    out = np.zeros((B, H, D), np.float64)
    lse = np.zeros((B, H), np.float64)
    _L().oracle_srswa_decode(B, H, D, n, cap, blk, _p(q), _p(pk), _p(pv), _p(prefix_len), _p(blk_idx),
                             _p(blk_logp), topk, _p(ring_k), _p(ring_v), _p(wp), _p(fill), float(scale),
                             _p(out), _p(lse))
    return out, lse


# ---------------------------------------------------------------- SR-SWA chunked prefill

def route_tokens(q_idx, kbar, prefix_len, topk: int = 16, idx_scale: float = 1.0, blk: int = BLOCK):
    """Per-token routes of a prefill chunk: q_idx fp32 [B][T][DI] against kbar [B][NBcap][DI].
    Returns (blk_idx int32 [B][T][topk], blk_logp fp64 [B][T][topk])."""
    q_idx = np.ascontiguousarray(q_idx, np.float32)
    kbar = np.ascontiguousarray(kbar, np.float64)
    prefix_len = _i32(prefix_len, "prefix_len")
    B, nb_cap, DI = kbar.shape
    if q_idx.ndim != 3 or q_idx.shape[0] != B or q_idx.shape[2] != DI:
        raise ValueError("q_idx shape")
    T = q_idx.shape[1]
    blk_idx = np.zeros((B, T, topk), np.int32)
    blk_logp = np.zeros((B, T, topk), np.float64)
    _L().oracle_route_tokens(B, T, nb_cap, DI, blk, _p(q_idx), _p(kbar), _p(prefix_len), float(idx_scale),
                             int(topk), _p(blk_idx), _p(blk_logp))
    return blk_idx, blk_logp


def srswa_prefill(q, k_out, v_out, pk, pv, prefix_len, blk_idx, blk_logp, scale, rows, n, ring_k=None, ring_v=None,
                  wp=None, fill=None, blk: int = BLOCK):
    """SR-SWA chunked prefill for the listed query rows, routes given ([B][T][topk]).
    Returns (out [B][H][R][D], lse [B][H][R])."""
    q = _u16(q, 4, "q")
    k_out = _u16(k_out, 4, "k_out")
    v_out = _u16(v_out, 4, "v_out")
    pk = _u16(pk, 4, "pk")
    pv = _u16(pv, 4, "pv")
    B, H, T, D = q.shape
    cap = pk.shape[2]
    prefix_len = _i32(prefix_len, "prefix_len")
    blk_idx = _i32(blk_idx, "blk_idx")
    blk_logp = np.ascontiguousarray(blk_logp, np.float64)
    if blk_idx.ndim != 3 or blk_idx.shape[:2] != (B, T):
        raise ValueError("blk_idx shape")
    topk = blk_idx.shape[2]
    rows = _i32(np.asarray(rows, np.int32), "rows")
    if rows.size and (rows.min() < 0 or rows.max() >= T):
        raise ValueError("row index out of range")
    if ring_k is not None:
        ring_k = _u16(ring_k, 4, "ring_k")
        ring_v = _u16(ring_v, 4, "ring_v")
        wp, fill = _i32(wp, "wp"), _i32(fill, "fill")
        if ring_k.shape[2] != n:
            raise ValueError("ring slots != n")
    R = rows.size
    out = np.zeros((B, H, R, D), np.float64)
    lse = np.zeros((B, H, R), np.float64)
    _L().oracle_srswa_prefill(B, H, D, int(n), cap, T, blk, _p(q), _p(k_out), _p(v_out), _p(pk), _p(pv),
                              _p(prefix_len), _p(blk_idx), _p(blk_logp), topk, _p(ring_k), _p(ring_v), _p(wp),
                              _p(fill), float(scale), _p(rows), R, _p(out), _p(lse))
    return out, lse


# ---------------------------------------------------------------- FP8 (e4m3) prefix

def e4m3_to_double(codes) -> np.ndarray:
    """Values of E4M3 codes (uint8 array), from the format's definition (NaN for 0x7f / 0xff)."""
    table = np.array([_L().oracle_e4m3_to_double(c) for c in range(256)], np.float64)
    return table[np.asarray(codes, np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """Nearest E4M3 codes of fp32 values (ties to even, saturating at 448, NaN -> 0x7f)."""
    x = np.ascontiguousarray(x, np.float32)
    out = np.zeros(x.shape, np.uint8)
    _L().oracle_e4m3_encode_array(x.size, _p(x), _p(out))
    return out


def quantize_prefix(x, prefix_len, blk: int = BLOCK):
    """E4M3 codes [B][H][cap][D] (uint8) and fp32 block scales [B][H][ceil(cap/blk)] of a bf16 prefix.

    Blocks past prefix_len are left at zero (codes) / zero (scales) here."""
    x = _u16(x, 4, "x")
    prefix_len = _i32(prefix_len, "prefix_len")
    B, H, cap, D = x.shape
    codes = np.zeros((B, H, cap, D), np.uint8)
    scales = np.zeros((B, H, (cap + blk - 1) // blk), np.float32)
    _L().oracle_quantize_prefix(B, H, D, cap, blk, _p(x), _p(prefix_len), _p(codes), _p(scales))
    return codes, scales


def _u8(a, ndim: int, name: str) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint8 or a.ndim != ndim:
        raise ValueError(f"{name}: expected uint8 with {ndim} dims, got {a.dtype} {a.shape}")
    return a


def rswa_decode_fp8(q, pk8, pv8, kscale, vscale, prefix_len, ring_k, ring_v, wp, fill, scale, blk: int = BLOCK):
    """R-SWA decode over an E4M3 prefix (code * block scale). Returns (out fp64 [B][H][D], lse fp64 [B][H])."""
    q = _u16(q, 3, "q")
    pk8, pv8 = _u8(pk8, 4, "pk8"), _u8(pv8, 4, "pv8")
    kscale = np.ascontiguousarray(kscale, np.float32)
    vscale = np.ascontiguousarray(vscale, np.float32)
    ring_k = _u16(ring_k, 4, "ring_k")
    ring_v = _u16(ring_v, 4, "ring_v")
    prefix_len, wp, fill = _i32(prefix_len, "prefix_len"), _i32(wp, "wp"), _i32(fill, "fill")
    B, H, D = q.shape
    cap = pk8.shape[2]
    n = ring_k.shape[2]
    out = np.zeros((B, H, D), np.float64)
    lse = np.zeros((B, H), np.float64)
    _L().oracle_rswa_decode_fp8(B, H, D, n, cap, blk, _p(q), _p(pk8), _p(pv8), _p(kscale), _p(vscale),
                                _p(prefix_len), _p(ring_k), _p(ring_v), _p(wp), _p(fill), float(scale), _p(out),
                                _p(lse))
    return out, lse


def srswa_decode_fp8(q, pk8, pv8, kscale, vscale, prefix_len, blk_idx, blk_logp, ring_k, ring_v, wp, fill, scale,
                     blk: int = BLOCK):
    """SR-SWA gathered-block decode over an E4M3 prefix. Returns (out fp64 [B][H][D], lse fp64 [B][H])."""
    q = _u16(q, 3, "q")
    pk8, pv8 = _u8(pk8, 4, "pk8"), _u8(pv8, 4, "pv8")
    kscale = np.ascontiguousarray(kscale, np.float32)
    vscale = np.ascontiguousarray(vscale, np.float32)
    ring_k = _u16(ring_k, 4, "ring_k")
    ring_v = _u16(ring_v, 4, "ring_v")
    prefix_len, wp, fill = _i32(prefix_len, "prefix_len"), _i32(wp, "wp"), _i32(fill, "fill")
    blk_idx = _i32(blk_idx, "blk_idx")
    blk_logp = np.ascontiguousarray(blk_logp, np.float64)
    B, H, D = q.shape
    topk = blk_idx.shape[1]
    cap = pk8.shape[2]
    n = ring_k.shape[2]
    out = np.zeros((B, H, D), np.float64)
    lse = np.zeros((B, H), np.float64)
    _L().oracle_srswa_decode_fp8(B, H, D, n, cap, blk, _p(q), _p(pk8), _p(pv8), _p(kscale), _p(vscale),
                                 _p(prefix_len), _p(blk_idx), _p(blk_logp), topk, _p(ring_k), _p(ring_v), _p(wp),
                                 _p(fill), float(scale), _p(out), _p(lse))
    return out, lse


# ---------------------------------------------------------------- FP8 ring

def fp8_ring(B: int, H: int, n: int, D: int = 128):
    """An empty FP8 ring: codes (K, V) uint8 [B][H][n][D] and row scales (K, V) f32 [B][H][n]."""
    return (np.zeros((B, H, n, D), np.uint8), np.zeros((B, H, n, D), np.uint8), np.ones((B, H, n), np.float32),
            np.ones((B, H, n), np.float32))


def append_fp8(rk8, rv8, rks, rvs, k_new, v_new, wp, fill):
    """Ring append into an FP8 ring (each written row quantised with its own scale), in place on
    the codes, scales, wp and fill. Returns slot_out [B]."""
    for name, a in (("rk8", rk8), ("rv8", rv8), ("rks", rks), ("rvs", rvs), ("wp", wp), ("fill", fill)):
        if not (isinstance(a, np.ndarray) and a.flags.c_contiguous):
            raise ValueError(f"{name} must be a C-contiguous numpy array (updated in place)")
    if rk8.dtype != np.uint8 or rks.dtype != np.float32 or wp.dtype != np.int32:
        raise TypeError("codes uint8, scales float32, wp / fill int32")
    B, H, n, D = rk8.shape
    k_new, v_new = _u16(k_new, 3, "k_new"), _u16(v_new, 3, "v_new")
    slot = np.zeros(B, np.int32)
    _L().oracle_append_fp8(B, H, n, D, _p(rk8), _p(rv8), _p(rks), _p(rvs), _p(k_new), _p(v_new), _p(wp), _p(fill),
                           _p(slot))
    return slot


def rswa_decode_fp8kv(q, pk8, pv8, kscale, vscale, prefix_len, rk8, rv8, rks, rvs, wp, fill, scale,
                      blk: int = BLOCK):
    """R-SWA decode over an E4M3 prefix (block scales) and an E4M3 ring (row scales).
    Returns (out fp64 [B][H][D], lse fp64 [B][H])."""
    q = _u16(q, 3, "q")
    pk8, pv8, rk8, rv8 = _u8(pk8, 4, "pk8"), _u8(pv8, 4, "pv8"), _u8(rk8, 4, "rk8"), _u8(rv8, 4, "rv8")
    kscale, vscale = np.ascontiguousarray(kscale, np.float32), np.ascontiguousarray(vscale, np.float32)
    rks, rvs = np.ascontiguousarray(rks, np.float32), np.ascontiguousarray(rvs, np.float32)
    prefix_len, wp, fill = _i32(prefix_len, "prefix_len"), _i32(wp, "wp"), _i32(fill, "fill")
    B, H, D = q.shape
    cap, n = pk8.shape[2], rk8.shape[2]
    out = np.zeros((B, H, D), np.float64)
    lse = np.zeros((B, H), np.float64)
    _L().oracle_rswa_decode_fp8kv(B, H, D, n, cap, blk, _p(q), _p(pk8), _p(pv8), _p(kscale), _p(vscale),
                                  _p(prefix_len), _p(rk8), _p(rv8), _p(rks), _p(rvs), _p(wp), _p(fill), float(scale),
                                  _p(out), _p(lse))
    return out, lse


def srswa_decode_fp8kv(q, pk8, pv8, kscale, vscale, prefix_len, blk_idx, blk_logp, rk8, rv8, rks, rvs, wp, fill,
                       scale, blk: int = BLOCK):
    """SR-SWA gathered-block decode over an E4M3 prefix and an E4M3 ring.
    Returns (out fp64 [B][H][D], lse fp64 [B][H])."""
    q = _u16(q, 3, "q")
    pk8, pv8, rk8, rv8 = _u8(pk8, 4, "pk8"), _u8(pv8, 4, "pv8"), _u8(rk8, 4, "rk8"), _u8(rv8, 4, "rv8")
    kscale, vscale = np.ascontiguousarray(kscale, np.float32), np.ascontiguousarray(vscale, np.float32)
    rks, rvs = np.ascontiguousarray(rks, np.float32), np.ascontiguousarray(rvs, np.float32)
    prefix_len, wp, fill = _i32(prefix_len, "prefix_len"), _i32(wp, "wp"), _i32(fill, "fill")
    blk_idx = _i32(blk_idx, "blk_idx")
    blk_logp = np.ascontiguousarray(blk_logp, np.float64)
    B, H, D = q.shape
    topk = blk_idx.shape[1]
    cap, n = pk8.shape[2], rk8.shape[2]
    out = np.zeros((B, H, D), np.float64)
    lse = np.zeros((B, H), np.float64)
    _L().oracle_srswa_decode_fp8kv(B, H, D, n, cap, blk, _p(q), _p(pk8), _p(pv8), _p(kscale), _p(vscale),
                                   _p(prefix_len), _p(blk_idx), _p(blk_logp), topk, _p(rk8), _p(rv8), _p(rks),
                                   _p(rvs), _p(wp), _p(fill), float(scale), _p(out), _p(lse))
    return out, lse


# ---------------------------------------------------------------- page2d rotary encoding

def bf16_round(x) -> np.ndarray:
    """Nearest bf16 bit patterns (uint16) of fp64 values, ties to even."""
    x = np.ascontiguousarray(x, np.float64)
    out = np.zeros(x.shape, np.uint16)
    _L().oracle_bf16_round_array(x.size, _p(x), _p(out))
    return out


def rope_page2d(x, tok_pos, page, base: float = 10000.0, page_mod: int = 2) -> np.ndarray:
    """page2d rotary encoding of bf16 rows x uint16 [..., H, D]; tok_pos / page int32 with the
    shape of x's leading dims (one token-axis and one page-axis position per row).
    Returns the exact rotation in fp64, shaped like x (readings: oracle_rope_page2d)."""
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16 or x.ndim < 2:
        raise TypeError("x: expected bf16 bit patterns as uint16 [..., H, D]")
    H, D = x.shape[-2:]
    if D % 2:
        raise ValueError("D must be even")
    lead = x.shape[:-2]
    tok_pos = _i32(np.asarray(tok_pos, np.int32), "tok_pos")
    page = _i32(np.asarray(page, np.int32), "page")
    if tok_pos.shape != lead or page.shape != lead:
        raise ValueError(f"positions must have shape {lead}")
    if page_mod < 0:
        raise ValueError("page_mod must be >= 0")
    rows = int(np.prod(lead)) if lead else 1
    out = np.zeros(x.shape, np.float64)
    _L().oracle_rope_page2d(rows, H, D, _p(x), _p(tok_pos), _p(page), float(base), int(page_mod), _p(out))
    return out


def kv_cache_bytes(ref_tokens: int, T: int, heads: int, head_dim: int, layers: int, bytes_per_elem: int,
                   window: int | None) -> int:
    """KV-cache bytes after T generated tokens.

    Cached tokens are L_m + T for full attention (window=None) and
    L_m + min(n, T) for R-SWA with window n ([R-SWA summary] §二.2); each token
    stores K and V for every head of every layer.
    """
    cached = ref_tokens + (T if window is None else min(window, T))
    return cached * 2 * heads * head_dim * bytes_per_elem * layers


def bf16_bits_to_f64(a: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to float64 exactly."""
    return (np.asarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
