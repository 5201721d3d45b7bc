"""ctypes binding of librswa.so: argument marshalling only.

Each function takes torch CUDA tensors, checks dtype/device/shape/contiguity,
and passes ``data_ptr()`` values and the CUDA stream handle to the C entry
point of the same name (declared in ``include/rswa.h``). Every step of the
computation runs in the library's kernels; there is no CPU or PyTorch
fallback: if the library is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# RSWA_LIBRARY selects another build of the same library (for example one
# compiled with different pipeline-depth constants); default: the in-tree build.
LIB_PATH = os.environ.get("RSWA_LIBRARY") or os.path.join(_PKG, "librswa.so")
_DEFAULT_LIB = os.path.join(_PKG, "librswa.so")

OP_DECODE = 1
OP_SRSWA_DECODE = 2
OP_ROUTE = 3
OP_PREFILL = 4
OP_SRSWA_ROUTED = 5

STATUS_NAMES = {0: "RSWA_OK", 1: "RSWA_ERR_INVALID", 2: "RSWA_ERR_UNSUPPORTED", 3: "RSWA_ERR_CUDA",
                5: "RSWA_ERR_DEVICE_CHECK"}
DEVICE_BAD_PREFIX_LEN = 0x1
DEVICE_BAD_RING_STATE = 0x2
DEVICE_BAD_BLOCK_IDX = 0x4
DEVICE_WAIT_TIMEOUT = 0x8
DEVICE_PIPELINE = 0x10

EXPORTED = ("rswa_last_error", "rswa_version", "rswa_workspace_bytes", "rswa_check_status", "rswa_append",
            "rswa_decode", "srswa_index_pool", "srswa_route", "srswa_decode", "rswa_decode_noalloc", "rswa_prefill",
            "rswa_quantize_prefix", "rswa_decode_fp8", "srswa_decode_fp8", "srswa_route_tokens", "srswa_prefill",
            "rswa_decode_append", "srswa_decode_append", "rswa_rope_page2d", "rswa_append_rope", "rswa_append_fp8",
            "rswa_decode_fp8kv", "srswa_decode_fp8kv", "rswa_test_arm_wait_timeout", "srswa_decode_routed",
            "srswa_step", "srswa_prefill_workspace_bytes", "rswa_decode_append_rope", "srswa_step_rope")


class RswaError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} -> {STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("ring", ctypes.c_int32), ("prefix_cap", ctypes.c_int64)]

    def __repr__(self):
        return (f"Dims(batch={self.batch}, heads={self.heads}, head_dim={self.head_dim}, ring={self.ring}, "
                f"prefix_cap={self.prefix_cap})")


class Rope(ctypes.Structure):
    """rswa_rope: the page2d encoding of a fused decode step (device position arrays)."""
    _fields_ = [("tok_pos", ctypes.c_void_p), ("page", ctypes.c_void_p), ("base", ctypes.c_double),
                ("page_mod", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def load(path: str | None = None):
    """Load librswa.so (building it first if the sources are newer). Raises if unavailable."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if path is None and p == _DEFAULT_LIB:
            from . import build as _build
            try:
                if not _build.up_to_date():
                    _build.build()
            except RuntimeError:
                if not os.path.exists(p):
                    raise
        if not os.path.exists(p):
            raise RuntimeError(f"librswa.so not found at {p}; run python -m long_context_decode_swa_b200.build")
        lib = ctypes.CDLL(p)
        P, I32, I64, F32, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        DP = ctypes.POINTER(Dims)
        RP = ctypes.POINTER(Rope)
        sig = {
            "rswa_last_error": ([], ctypes.c_char_p),
            "rswa_version": ([], I32),
            "rswa_workspace_bytes": ([DP, I32], SZ),
            "rswa_check_status": ([P, SZ, P, P], ctypes.c_int),
            "rswa_test_arm_wait_timeout": ([I32, I64], ctypes.c_int),
            "srswa_decode_routed": ([DP, P, P, P, F32, I32, P, P, P, P, P, P, P, F32, P, P, P, P, P, P, SZ, P],
                                    ctypes.c_int),
            "srswa_step": ([DP, P, P, P, P, P, F32, I32, P, P, P, P, P, P, P, P, F32, P, P, P, P, P, P, SZ, P],
                           ctypes.c_int),
            "srswa_prefill_workspace_bytes": ([DP, I32], SZ),
            "rswa_decode_append_rope": ([DP, RP, P, P, P, P, P, P, P, P, P, P, P, F32, P, P, P, SZ, P], ctypes.c_int),
            "srswa_step_rope": ([DP, RP, P, P, P, P, P, F32, I32, P, P, P, P, P, P, P, P, F32, P, P, P, P, P, P, SZ,
                                 P], ctypes.c_int),
            "rswa_append": ([DP, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "rswa_decode": ([DP, P, P, P, P, P, P, P, P, F32, P, P, P, SZ, P], ctypes.c_int),
            "srswa_index_pool": ([DP, P, P, P, P], ctypes.c_int),
            "srswa_route": ([DP, P, P, P, F32, I32, P, P, P, P, P, SZ, P], ctypes.c_int),
            "srswa_decode": ([DP, P, P, P, P, P, P, I32, P, P, P, P, F32, P, P, P, SZ, P], ctypes.c_int),
            "rswa_decode_noalloc": ([DP, P, P, P, P, P, P, P, P, F32, P, P, P, P], ctypes.c_int),
            "rswa_prefill": ([DP, I32, P, P, P, P, P, P, P, P, P, P, F32, P, P, I32, P, SZ, P], ctypes.c_int),
            "rswa_quantize_prefix": ([DP, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "rswa_decode_fp8": ([DP, P, P, P, P, P, P, P, P, P, P, F32, P, P, P, SZ, P], ctypes.c_int),
            "srswa_decode_fp8": ([DP, P, P, P, P, P, P, P, P, I32, P, P, P, P, F32, P, P, P, SZ, P], ctypes.c_int),
            "srswa_route_tokens": ([DP, I32, P, P, P, F32, I32, P, P, P, SZ, P], ctypes.c_int),
            "srswa_prefill": ([DP, I32, P, P, P, P, P, P, P, P, I32, P, P, P, P, F32, P, P, P, SZ, P], ctypes.c_int),
            "rswa_decode_append": ([DP, P, P, P, P, P, P, P, P, P, P, P, F32, P, P, P, SZ, P], ctypes.c_int),
            "srswa_decode_append": ([DP, P, P, P, P, P, P, P, P, I32, P, P, P, P, P, F32, P, P, P, SZ, P],
                                    ctypes.c_int),
            "rswa_rope_page2d": ([I64, I32, I32, P, P, P, P, P, P, ctypes.c_double, I32, P], ctypes.c_int),
            "rswa_append_rope": ([DP, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_double, I32, P, P], ctypes.c_int),
            "rswa_append_fp8": ([DP, P, P, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "rswa_decode_fp8kv": ([DP, P, P, P, P, P, P, P, P, P, P, P, P, F32, P, P, P, SZ, P], ctypes.c_int),
            "srswa_decode_fp8kv": ([DP, P, P, P, P, P, P, P, P, I32, P, P, P, P, P, P, F32, P, P, P, SZ, P],
                                   ctypes.c_int),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = res
        _lib = lib
        return lib


def _check(fn: str, code: int):
    if code != 0:
        raise RswaError(fn, code, load().rswa_last_error().decode())


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _want(t: torch.Tensor, name: str, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name}: must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def dims_of(pk: torch.Tensor, ring_k: torch.Tensor) -> Dims:
    B, H, cap, D = pk.shape
    return Dims(B, H, D, ring_k.shape[2], cap)


def workspace_bytes(dims: Dims, op: int) -> int:
    n = load().rswa_workspace_bytes(ctypes.byref(dims), op)
    if n == 0:
        raise RswaError("rswa_workspace_bytes", 1, load().rswa_last_error().decode())
    return int(n)


def new_workspace(dims: Dims, op: int, device=None) -> torch.Tensor:
    """A zero-filled workspace tensor (uint8) sized for `op` (see rswa_workspace_bytes)."""
    return torch.zeros(workspace_bytes(dims, op), dtype=torch.uint8, device=device or "cuda")


def route_workspace(batch: int, prefix_cap: int, device=None) -> torch.Tensor:
    """A zero-filled workspace for srswa_route over `batch` sequences of capacity `prefix_cap`."""
    return new_workspace(Dims(batch, 1, 128, 1, prefix_cap), OP_ROUTE, device)


def test_arm_wait_timeout(drop_tile: int, wait_limit_ns: int) -> None:
    """Test hook: the next decode-family call of this thread drops CTA 0's tile `drop_tile`
    (its bounded wait then runs out) and waits at most `wait_limit_ns` (see rswa.h)."""
    _check("rswa_test_arm_wait_timeout", load().rswa_test_arm_wait_timeout(int(drop_tile), int(wait_limit_ns)))


def check_status(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise, read and clear the device status word; returns it (0 = clean)."""
    st = ctypes.c_int32(0)
    code = load().rswa_check_status(_ptr(workspace), workspace.numel() * workspace.element_size(),
                                    ctypes.byref(st), _stream(stream))
    if code not in (0, 5):
        _check("rswa_check_status", code)
    return int(st.value)


def rswa_append(ring_k, ring_v, k_new, v_new, wp, fill, slot_out=None, status=None, stream=None):
    B, H, n, D = ring_k.shape
    _want(ring_k, "ring_k", torch.bfloat16)
    _want(ring_v, "ring_v", torch.bfloat16, ring_k.shape)
    _want(k_new, "k_new", torch.bfloat16, (B, H, D))
    _want(v_new, "v_new", torch.bfloat16, (B, H, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    if slot_out is not None:
        _want(slot_out, "slot_out", torch.int32, (B,))
    if status is not None:
        _want(status, "status", status.dtype)
    dims = Dims(B, H, D, n, 0)
    _check("rswa_append", load().rswa_append(ctypes.byref(dims), _ptr(ring_k), _ptr(ring_v), _ptr(k_new), _ptr(v_new),
                                             _ptr(wp), _ptr(fill), _ptr(slot_out), _ptr(status), _stream(stream)))


def rswa_rope_page2d(q, tok_pos, page, q_out=None, k=None, k_out=None, base: float = 10000.0, page_mod: int = 2,
                     stream=None):
    """page2d rotary encoding of q (and k) bf16 [..., H, D], one token per leading index with
    positions tok_pos / page (int32, shaped like the leading dims). q_out / k_out default to
    in place. Returns (q_out, k_out)."""
    if q.dim() < 2:
        raise ValueError("q: expected [..., H, D]")
    H, D = q.shape[-2:]
    lead = tuple(q.shape[:-2])
    _want(q, "q", torch.bfloat16)
    q_out = q if q_out is None else _want(q_out, "q_out", torch.bfloat16, q.shape)
    if k is not None:
        _want(k, "k", torch.bfloat16, q.shape)
        k_out = k if k_out is None else _want(k_out, "k_out", torch.bfloat16, q.shape)
    elif k_out is not None:
        raise ValueError("k_out given without k")
    _want(tok_pos, "tok_pos", torch.int32, lead)
    _want(page, "page", torch.int32, lead)
    rows = q.numel() // (H * D) if q.numel() else 0
    _check("rswa_rope_page2d", load().rswa_rope_page2d(rows, H, D, _ptr(q), _ptr(q_out), _ptr(k), _ptr(k_out),
                                                       _ptr(tok_pos), _ptr(page), float(base), int(page_mod),
                                                       _stream(stream)))
    return q_out, k_out


def rswa_append_rope(ring_k, ring_v, k_new, v_new, wp, fill, q, tok_pos, page, q_out=None, base: float = 10000.0,
                     page_mod: int = 2, slot_out=None, status=None, stream=None):
    """rswa_append with k_new page2d-encoded on its way into the ring and q encoded into q_out
    (default: in place), one launch. Returns q_out."""
    B, H, n, D = ring_k.shape
    _want(ring_k, "ring_k", torch.bfloat16)
    _want(ring_v, "ring_v", torch.bfloat16, ring_k.shape)
    _want(k_new, "k_new", torch.bfloat16, (B, H, D))
    _want(v_new, "v_new", torch.bfloat16, (B, H, D))
    _want(q, "q", torch.bfloat16, (B, H, D))
    q_out = q if q_out is None else _want(q_out, "q_out", torch.bfloat16, (B, H, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    _want(tok_pos, "tok_pos", torch.int32, (B,))
    _want(page, "page", torch.int32, (B,))
    if slot_out is not None:
        _want(slot_out, "slot_out", torch.int32, (B,))
    if status is not None:
        _want(status, "status", status.dtype)
    dims = Dims(B, H, D, n, 0)
    _check("rswa_append_rope", load().rswa_append_rope(ctypes.byref(dims), _ptr(ring_k), _ptr(ring_v), _ptr(k_new),
                                                       _ptr(v_new), _ptr(wp), _ptr(fill), _ptr(slot_out), _ptr(q),
                                                       _ptr(q_out), _ptr(tok_pos), _ptr(page), float(base),
                                                       int(page_mod), _ptr(status), _stream(stream)))
    return q_out


def rswa_decode(q, pk, pv, prefix_len, ring_k, ring_v, wp, fill, out, workspace, lse=None, scale=None, stream=None):
    B, H, cap, D = pk.shape
    n = ring_k.shape[2]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(pk, "pk", torch.bfloat16)
    _want(pv, "pv", torch.bfloat16, pk.shape)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
    _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("rswa_decode", load().rswa_decode(ctypes.byref(dims), _ptr(q), _ptr(pk), _ptr(pv), _ptr(prefix_len),
                                             _ptr(ring_k), _ptr(ring_v), _ptr(wp), _ptr(fill), scale, _ptr(out),
                                             _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))


def srswa_index_pool(k_idx, prefix_len, kbar, heads: int = 1, stream=None):
    B, cap, DI = k_idx.shape
    _want(k_idx, "k_idx", torch.bfloat16)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(kbar, "kbar", torch.float32, (B, (cap + 31) // 32, DI))
    if DI != 32:
        raise ValueError("index dim must be 32")
    dims = Dims(B, heads, 128, 1, cap)
    _check("srswa_index_pool", load().srswa_index_pool(ctypes.byref(dims), _ptr(k_idx), _ptr(prefix_len), _ptr(kbar),
                                                       _stream(stream)))


def srswa_route(q_idx, kbar, prefix_len, blk_idx, blk_logp, workspace, probs=None, tau=None, idx_scale=1.0,
                prefix_cap: int | None = None, stream=None):
    B, nb_cap, DI = kbar.shape
    topk = blk_idx.shape[1]
    _want(q_idx, "q_idx", torch.float32, (B, DI))
    _want(kbar, "kbar", torch.float32)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(blk_idx, "blk_idx", torch.int32, (B, topk))
    _want(blk_logp, "blk_logp", torch.float32, (B, topk))
    if probs is not None:
        _want(probs, "probs", torch.float32, (B, nb_cap))
    if tau is not None:
        _want(tau, "tau", torch.float32, (B,))
    _want(workspace, "workspace", torch.uint8)
    cap = nb_cap * 32 if prefix_cap is None else int(prefix_cap)
    if (cap + 31) // 32 != nb_cap:
        raise ValueError("prefix_cap does not match kbar's block count")
    dims = Dims(B, 1, 128, 1, cap)
    _check("srswa_route", load().srswa_route(ctypes.byref(dims), _ptr(q_idx), _ptr(kbar), _ptr(prefix_len),
                                             float(idx_scale), topk, _ptr(blk_idx), _ptr(blk_logp), _ptr(probs),
                                             _ptr(tau), _ptr(workspace), workspace.numel(), _stream(stream)))


def srswa_decode(q, pk, pv, prefix_len, blk_idx, blk_logp, ring_k, ring_v, wp, fill, out, workspace, lse=None,
                 scale=None, stream=None):
    B, H, cap, D = pk.shape
    n = ring_k.shape[2]
    topk = blk_idx.shape[1]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(pk, "pk", torch.bfloat16)
    _want(pv, "pv", torch.bfloat16, pk.shape)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(blk_idx, "blk_idx", torch.int32, (B, topk))
    _want(blk_logp, "blk_logp", torch.float32, (B, topk))
    _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
    _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("srswa_decode", load().srswa_decode(ctypes.byref(dims), _ptr(q), _ptr(pk), _ptr(pv), _ptr(prefix_len),
                                               _ptr(blk_idx), _ptr(blk_logp), topk, _ptr(ring_k), _ptr(ring_v),
                                               _ptr(wp), _ptr(fill), scale, _ptr(out), _ptr(lse), _ptr(workspace),
                                               workspace.numel(), _stream(stream)))


def fp8_prefix_buffers(pk: torch.Tensor):
    """Empty E4M3 code tensors (uint8, pk's shape) and f32 block-scale tensors [B][H][ceil(cap/32)] for K and V."""
    B, H, cap, D = pk.shape
    nb = (cap + 31) // 32
    dev = pk.device
    return (torch.empty((B, H, cap, D), dtype=torch.uint8, device=dev),
            torch.empty((B, H, cap, D), dtype=torch.uint8, device=dev),
            torch.zeros((B, H, nb), dtype=torch.float32, device=dev),
            torch.zeros((B, H, nb), dtype=torch.float32, device=dev))


def rswa_quantize_prefix(pk, pv, prefix_len, pk8, pv8, k_scale, v_scale, status=None, stream=None):
    B, H, cap, D = pk.shape
    _want(pk, "pk", torch.bfloat16)
    _want(pv, "pv", torch.bfloat16, pk.shape)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(pk8, "pk8", torch.uint8, pk.shape)
    _want(pv8, "pv8", torch.uint8, pk.shape)
    nb = (cap + 31) // 32
    _want(k_scale, "k_scale", torch.float32, (B, H, nb))
    _want(v_scale, "v_scale", torch.float32, (B, H, nb))
    dims = Dims(B, H, D, 1, cap)
    _check("rswa_quantize_prefix", load().rswa_quantize_prefix(ctypes.byref(dims), _ptr(pk), _ptr(pv),
                                                               _ptr(prefix_len), _ptr(pk8), _ptr(pv8),
                                                               _ptr(k_scale), _ptr(v_scale), _ptr(status),
                                                               _stream(stream)))


def _want_fp8_prefix(pk8, pv8, k_scale, v_scale):
    B, H, cap, D = pk8.shape
    _want(pk8, "pk8", torch.uint8)
    _want(pv8, "pv8", torch.uint8, pk8.shape)
    _want(k_scale, "k_scale", torch.float32, (B, H, (cap + 31) // 32))
    _want(v_scale, "v_scale", torch.float32, (B, H, (cap + 31) // 32))
    return B, H, cap, D


def rswa_decode_fp8(q, pk8, pv8, k_scale, v_scale, prefix_len, ring_k, ring_v, wp, fill, out, workspace, lse=None,
                    scale=None, stream=None):
    B, H, cap, D = _want_fp8_prefix(pk8, pv8, k_scale, v_scale)
    n = ring_k.shape[2]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
    _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("rswa_decode_fp8", load().rswa_decode_fp8(ctypes.byref(dims), _ptr(q), _ptr(pk8), _ptr(pv8),
                                                     _ptr(k_scale), _ptr(v_scale), _ptr(prefix_len), _ptr(ring_k),
                                                     _ptr(ring_v), _ptr(wp), _ptr(fill), scale, _ptr(out),
                                                     _ptr(lse), _ptr(workspace), workspace.numel(),
                                                     _stream(stream)))


def fp8_ring_buffers(ring_shape, device=None):
    """An FP8 ring: E4M3 code tensors (uint8) [B][H][n][D] and f32 row-scale tensors [B][H][n] for K and V."""
    B, H, n, D = ring_shape
    dev = device or "cuda"
    return (torch.zeros((B, H, n, D), dtype=torch.uint8, device=dev),
            torch.zeros((B, H, n, D), dtype=torch.uint8, device=dev),
            torch.ones((B, H, n), dtype=torch.float32, device=dev),
            torch.ones((B, H, n), dtype=torch.float32, device=dev))


def _want_fp8_ring(ring_k8, ring_v8, ring_kscale, ring_vscale):
    B, H, n, D = ring_k8.shape
    _want(ring_k8, "ring_k8", torch.uint8)
    _want(ring_v8, "ring_v8", torch.uint8, (B, H, n, D))
    _want(ring_kscale, "ring_kscale", torch.float32, (B, H, n))
    _want(ring_vscale, "ring_vscale", torch.float32, (B, H, n))
    return B, H, n, D


def rswa_append_fp8(ring_k8, ring_v8, ring_kscale, ring_vscale, k_new, v_new, wp, fill, slot_out=None, status=None,
                    stream=None):
    """rswa_append into an FP8 ring (each written row quantised with its own scale)."""
    B, H, n, D = _want_fp8_ring(ring_k8, ring_v8, ring_kscale, ring_vscale)
    _want(k_new, "k_new", torch.bfloat16, (B, H, D))
    _want(v_new, "v_new", torch.bfloat16, (B, H, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    if slot_out is not None:
        _want(slot_out, "slot_out", torch.int32, (B,))
    if status is not None:
        _want(status, "status", status.dtype)
    dims = Dims(B, H, D, n, 0)
    _check("rswa_append_fp8", load().rswa_append_fp8(ctypes.byref(dims), _ptr(ring_k8), _ptr(ring_v8),
                                                     _ptr(ring_kscale), _ptr(ring_vscale), _ptr(k_new), _ptr(v_new),
                                                     _ptr(wp), _ptr(fill), _ptr(slot_out), _ptr(status),
                                                     _stream(stream)))


def rswa_decode_fp8kv(q, pk8, pv8, k_scale, v_scale, prefix_len, ring_k8, ring_v8, ring_kscale, ring_vscale, wp, fill,
                      out, workspace, lse=None, scale=None, stream=None):
    """rswa_decode_fp8 with the ring read as E4M3 codes and row scales."""
    B, H, cap, D = _want_fp8_prefix(pk8, pv8, k_scale, v_scale)
    n = _want_fp8_ring(ring_k8, ring_v8, ring_kscale, ring_vscale)[2]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("rswa_decode_fp8kv", load().rswa_decode_fp8kv(ctypes.byref(dims), _ptr(q), _ptr(pk8), _ptr(pv8),
                                                         _ptr(k_scale), _ptr(v_scale), _ptr(prefix_len),
                                                         _ptr(ring_k8), _ptr(ring_v8), _ptr(ring_kscale),
                                                         _ptr(ring_vscale), _ptr(wp), _ptr(fill), scale, _ptr(out),
                                                         _ptr(lse), _ptr(workspace), workspace.numel(),
                                                         _stream(stream)))


def srswa_decode_fp8kv(q, pk8, pv8, k_scale, v_scale, prefix_len, blk_idx, blk_logp, ring_k8, ring_v8, ring_kscale,
                       ring_vscale, wp, fill, out, workspace, lse=None, scale=None, stream=None):
    """srswa_decode_fp8 with the ring read as E4M3 codes and row scales."""
    B, H, cap, D = _want_fp8_prefix(pk8, pv8, k_scale, v_scale)
    n = _want_fp8_ring(ring_k8, ring_v8, ring_kscale, ring_vscale)[2]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(blk_idx, "blk_idx", torch.int32)
    topk = blk_idx.shape[1]
    _want(blk_logp, "blk_logp", torch.float32, (B, topk))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("srswa_decode_fp8kv", load().srswa_decode_fp8kv(ctypes.byref(dims), _ptr(q), _ptr(pk8), _ptr(pv8),
                                                           _ptr(k_scale), _ptr(v_scale), _ptr(prefix_len),
                                                           _ptr(blk_idx), _ptr(blk_logp), topk, _ptr(ring_k8),
                                                           _ptr(ring_v8), _ptr(ring_kscale), _ptr(ring_vscale),
                                                           _ptr(wp), _ptr(fill), scale, _ptr(out), _ptr(lse),
                                                           _ptr(workspace), workspace.numel(), _stream(stream)))


def srswa_decode_fp8(q, pk8, pv8, k_scale, v_scale, prefix_len, blk_idx, blk_logp, ring_k, ring_v, wp, fill, out,
                     workspace, lse=None, scale=None, stream=None):
    B, H, cap, D = _want_fp8_prefix(pk8, pv8, k_scale, v_scale)
    n = ring_k.shape[2]
    topk = blk_idx.shape[1]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(blk_idx, "blk_idx", torch.int32, (B, topk))
    _want(blk_logp, "blk_logp", torch.float32, (B, topk))
    _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
    _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("srswa_decode_fp8", load().srswa_decode_fp8(ctypes.byref(dims), _ptr(q), _ptr(pk8), _ptr(pv8),
                                                       _ptr(k_scale), _ptr(v_scale), _ptr(prefix_len),
                                                       _ptr(blk_idx), _ptr(blk_logp), topk, _ptr(ring_k),
                                                       _ptr(ring_v), _ptr(wp), _ptr(fill), scale, _ptr(out),
                                                       _ptr(lse), _ptr(workspace), workspace.numel(),
                                                       _stream(stream)))


def rswa_decode_append(q, k_new, v_new, pk, pv, prefix_len, ring_k, ring_v, wp, fill, out, workspace, lse=None,
                       slot_out=None, scale=None, stream=None):
    """rswa_append + rswa_decode in one launch (same results; wp / fill / ring updated)."""
    B, H, cap, D = pk.shape
    n = ring_k.shape[2]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(k_new, "k_new", torch.bfloat16, (B, H, D))
    _want(v_new, "v_new", torch.bfloat16, (B, H, D))
    _want(pk, "pk", torch.bfloat16)
    _want(pv, "pv", torch.bfloat16, pk.shape)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
    _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    if slot_out is not None:
        _want(slot_out, "slot_out", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("rswa_decode_append", load().rswa_decode_append(ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new),
                                                           _ptr(pk), _ptr(pv), _ptr(prefix_len), _ptr(ring_k),
                                                           _ptr(ring_v), _ptr(wp), _ptr(fill), _ptr(slot_out), scale,
                                                           _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                                           _stream(stream)))


def _rope_arg(tok_pos, page, base, page_mod, B: int) -> Rope:
    _want(tok_pos, "tok_pos", torch.int32, (B,))
    _want(page, "page", torch.int32, (B,))
    return Rope(_ptr(tok_pos), _ptr(page), float(base), int(page_mod))


def rswa_decode_append_rope(q, k_new, v_new, pk, pv, prefix_len, ring_k, ring_v, wp, fill, tok_pos, page, out,
                            workspace, lse=None, slot_out=None, base: float = 10000.0, page_mod: int = 2, scale=None,
                            stream=None):
    """rswa_decode_append with q and k_new page2d-encoded inside the same launch (tok_pos, page:
    int32 [B], this step's positions)."""
    B, H, cap, D = pk.shape
    n = ring_k.shape[2]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(k_new, "k_new", torch.bfloat16, (B, H, D))
    _want(v_new, "v_new", torch.bfloat16, (B, H, D))
    _want(pk, "pk", torch.bfloat16)
    _want(pv, "pv", torch.bfloat16, pk.shape)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
    _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    if slot_out is not None:
        _want(slot_out, "slot_out", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    rope = _rope_arg(tok_pos, page, base, page_mod, B)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("rswa_decode_append_rope", load().rswa_decode_append_rope(
        ctypes.byref(dims), ctypes.byref(rope), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(pk), _ptr(pv),
        _ptr(prefix_len), _ptr(ring_k), _ptr(ring_v), _ptr(wp), _ptr(fill), _ptr(slot_out), scale, _ptr(out),
        _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))


def srswa_decode_append(q, k_new, v_new, pk, pv, prefix_len, blk_idx, blk_logp, ring_k, ring_v, wp, fill, out,
                        workspace, lse=None, slot_out=None, scale=None, stream=None):
    """rswa_append + srswa_decode in one launch (same results; wp / fill / ring updated)."""
    B, H, cap, D = pk.shape
    n = ring_k.shape[2]
    topk = blk_idx.shape[1]
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(k_new, "k_new", torch.bfloat16, (B, H, D))
    _want(v_new, "v_new", torch.bfloat16, (B, H, D))
    _want(pk, "pk", torch.bfloat16)
    _want(pv, "pv", torch.bfloat16, pk.shape)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(blk_idx, "blk_idx", torch.int32, (B, topk))
    _want(blk_logp, "blk_logp", torch.float32, (B, topk))
    _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
    _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    if slot_out is not None:
        _want(slot_out, "slot_out", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("srswa_decode_append", load().srswa_decode_append(ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new),
                                                             _ptr(pk), _ptr(pv), _ptr(prefix_len), _ptr(blk_idx),
                                                             _ptr(blk_logp), topk, _ptr(ring_k), _ptr(ring_v),
                                                             _ptr(wp), _ptr(fill), _ptr(slot_out), scale, _ptr(out),
                                                             _ptr(lse), _ptr(workspace), workspace.numel(),
                                                             _stream(stream)))


def srswa_route_tokens(q_idx, kbar, prefix_len, blk_idx, blk_logp, workspace, idx_scale=1.0, prefix_cap=None,
                       stream=None):
    """Per-token routes of a chunk: q_idx f32 [B][T][32] -> blk_idx int32 / blk_logp f32 [B][T][topk]."""
    B, nb_cap, DI = kbar.shape
    T = q_idx.shape[1]
    topk = blk_idx.shape[2]
    _want(q_idx, "q_idx", torch.float32, (B, T, DI))
    _want(kbar, "kbar", torch.float32)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(blk_idx, "blk_idx", torch.int32, (B, T, topk))
    _want(blk_logp, "blk_logp", torch.float32, (B, T, topk))
    _want(workspace, "workspace", torch.uint8)
    cap = nb_cap * 32 if prefix_cap is None else int(prefix_cap)
    dims = Dims(B, 1, 128, 1, cap)
    _check("srswa_route_tokens", load().srswa_route_tokens(ctypes.byref(dims), T, _ptr(q_idx), _ptr(kbar),
                                                           _ptr(prefix_len), float(idx_scale), topk, _ptr(blk_idx),
                                                           _ptr(blk_logp), _ptr(workspace), workspace.numel(),
                                                           _stream(stream)))


def srswa_prefill_workspace(batch: int, heads: int, T: int, prefix_cap: int, ring: int = 128, device=None):
    """A zero-filled workspace for srswa_prefill over `batch` x `heads` chunks of T queries."""
    dims = Dims(batch, heads, 128, ring, prefix_cap)
    n = load().srswa_prefill_workspace_bytes(ctypes.byref(dims), int(T))
    if n == 0:
        raise RswaError("srswa_prefill_workspace_bytes", 1, load().rswa_last_error().decode())
    return torch.zeros(int(n), dtype=torch.uint8, device=device or "cuda")


def srswa_prefill(q, k_out, v_out, pk, pv, prefix_len, blk_idx, blk_logp, out, workspace, lse=None, ring_k=None,
                  ring_v=None, wp=None, fill=None, scale=None, ring: int = 128, stream=None):
    """SR-SWA chunked prefill of T queries per (sequence, head), routes given per token.
    workspace: srswa_prefill_workspace(B, H, T, prefix_cap)."""
    B, H, T, D = q.shape
    cap = pk.shape[2]
    topk = blk_idx.shape[2]
    _want(q, "q", torch.bfloat16, (B, H, T, D))
    _want(k_out, "k_out", torch.bfloat16, (B, H, T, D))
    _want(v_out, "v_out", torch.bfloat16, (B, H, T, D))
    _want(pk, "pk", torch.bfloat16, (B, H, cap, D))
    _want(pv, "pv", torch.bfloat16, (B, H, cap, D))
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(blk_idx, "blk_idx", torch.int32, (B, T, topk))
    _want(blk_logp, "blk_logp", torch.float32, (B, T, topk))
    _want(out, "out", torch.float32, (B, H, T, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H, T))
    n = ring
    if ring_k is not None:
        n = ring_k.shape[2]
        _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
        _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
        _want(wp, "wp", torch.int32, (B,))
        _want(fill, "fill", torch.int32, (B,))
    _want(workspace, "workspace", torch.uint8)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("srswa_prefill", load().srswa_prefill(ctypes.byref(dims), T, _ptr(q), _ptr(k_out), _ptr(v_out), _ptr(pk),
                                                 _ptr(pv), _ptr(prefix_len), _ptr(blk_idx), _ptr(blk_logp), topk,
                                                 _ptr(ring_k), _ptr(ring_v), _ptr(wp), _ptr(fill), scale, _ptr(out),
                                                 _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))


def rswa_prefill(q, k_out, v_out, pk, pv, prefix_len, out, workspace, lse=None, ring_k=None, ring_v=None, wp=None,
                 fill=None, write_ring=False, scale=None, ring: int | None = None, stream=None):
    """Chunked R-SWA prefill. q/k_out/v_out bf16 [B][H][T][D]; out f32 [B][H][T][D]."""
    B, H, T, D = q.shape
    cap = pk.shape[2]
    _want(q, "q", torch.bfloat16)
    _want(k_out, "k_out", torch.bfloat16, q.shape)
    _want(v_out, "v_out", torch.bfloat16, q.shape)
    _want(pk, "pk", torch.bfloat16, (B, H, cap, D))
    _want(pv, "pv", torch.bfloat16, (B, H, cap, D))
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(out, "out", torch.float32, (B, H, T, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H, T))
    _want(workspace, "workspace", torch.uint8)
    if ring_k is not None:
        n = ring_k.shape[2]
        _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
        _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
        _want(wp, "wp", torch.int32, (B,))
        _want(fill, "fill", torch.int32, (B,))
    else:
        if ring is None:
            raise ValueError("without a ring tensor, pass the window length as ring=n")
        n = int(ring)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("rswa_prefill", load().rswa_prefill(ctypes.byref(dims), T, _ptr(q), _ptr(k_out), _ptr(v_out), _ptr(pk),
                                               _ptr(pv), _ptr(prefix_len), _ptr(ring_k), _ptr(ring_v), _ptr(wp),
                                               _ptr(fill), scale, _ptr(out), _ptr(lse), 1 if write_ring else 0,
                                               _ptr(workspace), workspace.numel(), _stream(stream)))


def _want_routed(q, q_idx, kbar, pk, pv, prefix_len, ring_k, ring_v, wp, fill, blk_idx, blk_logp, tau, out, lse,
                 workspace):
    B, H, cap, D = pk.shape
    n = ring_k.shape[2]
    topk = blk_idx.shape[1]
    nb_cap = (cap + 31) // 32
    _want(q, "q", torch.bfloat16, (B, H, D))
    _want(q_idx, "q_idx", torch.float32, (B, 32))
    _want(kbar, "kbar", torch.float32, (B, nb_cap, 32))
    _want(pk, "pk", torch.bfloat16)
    _want(pv, "pv", torch.bfloat16, pk.shape)
    _want(prefix_len, "prefix_len", torch.int32, (B,))
    _want(ring_k, "ring_k", torch.bfloat16, (B, H, n, D))
    _want(ring_v, "ring_v", torch.bfloat16, (B, H, n, D))
    _want(wp, "wp", torch.int32, (B,))
    _want(fill, "fill", torch.int32, (B,))
    _want(blk_idx, "blk_idx", torch.int32, (B, topk))
    _want(blk_logp, "blk_logp", torch.float32, (B, topk))
    if tau is not None:
        _want(tau, "tau", torch.float32, (B,))
    _want(out, "out", torch.float32, (B, H, D))
    if lse is not None:
        _want(lse, "lse", torch.float32, (B, H))
    _want(workspace, "workspace", torch.uint8)
    return B, H, cap, D, n, topk


def srswa_decode_routed(q, q_idx, kbar, pk, pv, prefix_len, ring_k, ring_v, wp, fill, blk_idx, blk_logp, out,
                        workspace, lse=None, tau=None, idx_scale=1.0, scale=None, stream=None):
    """srswa_route + srswa_decode in one launch: the route (blk_idx, blk_logp, tau) is an output.
    workspace: new_workspace(dims, OP_SRSWA_ROUTED)."""
    B, H, cap, D, n, topk = _want_routed(q, q_idx, kbar, pk, pv, prefix_len, ring_k, ring_v, wp, fill, blk_idx,
                                         blk_logp, tau, out, lse, workspace)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("srswa_decode_routed", load().srswa_decode_routed(
        ctypes.byref(dims), _ptr(q), _ptr(q_idx), _ptr(kbar), float(idx_scale), topk, _ptr(pk), _ptr(pv),
        _ptr(prefix_len), _ptr(ring_k), _ptr(ring_v), _ptr(wp), _ptr(fill), scale, _ptr(blk_idx), _ptr(blk_logp),
        _ptr(tau), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))


def srswa_step(q, k_new, v_new, q_idx, kbar, pk, pv, prefix_len, ring_k, ring_v, wp, fill, blk_idx, blk_logp, out,
               workspace, lse=None, tau=None, slot_out=None, idx_scale=1.0, scale=None, stream=None):
    """The whole SR-SWA decode step in one launch: rswa_append + srswa_route + srswa_decode.
    workspace: new_workspace(dims, OP_SRSWA_ROUTED)."""
    B, H, cap, D, n, topk = _want_routed(q, q_idx, kbar, pk, pv, prefix_len, ring_k, ring_v, wp, fill, blk_idx,
                                         blk_logp, tau, out, lse, workspace)
    _want(k_new, "k_new", torch.bfloat16, (B, H, D))
    _want(v_new, "v_new", torch.bfloat16, (B, H, D))
    if slot_out is not None:
        _want(slot_out, "slot_out", torch.int32, (B,))
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("srswa_step", load().srswa_step(
        ctypes.byref(dims), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_idx), _ptr(kbar), float(idx_scale), topk,
        _ptr(pk), _ptr(pv), _ptr(prefix_len), _ptr(ring_k), _ptr(ring_v), _ptr(wp), _ptr(fill), _ptr(slot_out), scale,
        _ptr(blk_idx), _ptr(blk_logp), _ptr(tau), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream)))


def srswa_step_rope(q, k_new, v_new, q_idx, kbar, pk, pv, prefix_len, ring_k, ring_v, wp, fill, tok_pos, page,
                    blk_idx, blk_logp, out, workspace, lse=None, tau=None, slot_out=None, base: float = 10000.0,
                    page_mod: int = 2, idx_scale=1.0, scale=None, stream=None):
    """srswa_step with q and k_new page2d-encoded inside the same launch (tok_pos, page: int32 [B],
    this step's positions; the router's q_idx is not encoded). workspace: new_workspace(dims,
    OP_SRSWA_ROUTED)."""
    B, H, cap, D, n, topk = _want_routed(q, q_idx, kbar, pk, pv, prefix_len, ring_k, ring_v, wp, fill, blk_idx,
                                         blk_logp, tau, out, lse, workspace)
    _want(k_new, "k_new", torch.bfloat16, (B, H, D))
    _want(v_new, "v_new", torch.bfloat16, (B, H, D))
    if slot_out is not None:
        _want(slot_out, "slot_out", torch.int32, (B,))
    rope = _rope_arg(tok_pos, page, base, page_mod, B)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dims = Dims(B, H, D, n, cap)
    _check("srswa_step_rope", load().srswa_step_rope(
        ctypes.byref(dims), ctypes.byref(rope), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(q_idx), _ptr(kbar),
        float(idx_scale), topk, _ptr(pk), _ptr(pv), _ptr(prefix_len), _ptr(ring_k), _ptr(ring_v), _ptr(wp),
        _ptr(fill), _ptr(slot_out), scale, _ptr(blk_idx), _ptr(blk_logp), _ptr(tau), _ptr(out), _ptr(lse),
        _ptr(workspace), workspace.numel(), _stream(stream)))
