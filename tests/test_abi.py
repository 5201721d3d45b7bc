"""The C-ABI library loads, exports every entry point include/rswa.h declares,
and rejects bad arguments on the host before launching anything (these calls
never reach a CUDA launch, so they run without a GPU)."""
import ctypes
import os
import re

import pytest

import long_context_decode_swa_b200 as rswa
from long_context_decode_swa_b200.binding import Dims

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
INVALID, UNSUPPORTED = 1, 2
A = ctypes.c_void_p(0x10000)      # 16-byte aligned stand-in pointers: never dereferenced by a
A2 = ctypes.c_void_p(0x20000)     # call that fails validation
MIS = ctypes.c_void_p(0x10008)    # misaligned


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "rswa.h"), encoding="utf-8").read()
    return sorted(set(re.findall(r"RSWA_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


def test_header_declares_the_documented_api():
    assert declared_symbols() == sorted(rswa.EXPORTED)


def test_library_exports_every_declared_symbol():
    lib = rswa.load()
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.rswa_version() == 5


def _err():
    return rswa.load().rswa_last_error().decode()


def test_workspace_bytes_rejects_bad_dims():
    lib = rswa.load()
    assert lib.rswa_workspace_bytes(ctypes.byref(Dims(4, 16, 64, 128, 100)), 1) == 0
    assert "head_dim" in _err()
    assert lib.rswa_workspace_bytes(ctypes.byref(Dims(0, 16, 128, 128, 100)), 1) == 0
    assert lib.rswa_workspace_bytes(ctypes.byref(Dims(4, 16, 128, 128, 100)), 99) == 0
    assert lib.rswa_workspace_bytes(ctypes.byref(Dims(4, 16, 128, 128, 100)), 1) >= 256


def test_decode_validation():
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 64)
    ws = lib.rswa_workspace_bytes(ctypes.byref(d), 1)
    args = lambda **kw: [ctypes.byref(kw.get("dims", d)), kw.get("q", A), A, A, A, A, A, A, A,
                         ctypes.c_float(kw.get("scale", 0.088)), kw.get("out", A), None, A,
                         ctypes.c_size_t(kw.get("ws", ws)), None]
    assert lib.rswa_decode(*args(q=None)) == INVALID and "q must not be NULL" in _err()
    assert lib.rswa_decode(*args(q=MIS)) == INVALID and "aligned" in _err()
    assert lib.rswa_decode(*args(out=None)) == INVALID
    assert lib.rswa_decode(*args(scale=0.0)) == INVALID and "scale" in _err()
    assert lib.rswa_decode(*args(scale=float("nan"))) == INVALID
    assert lib.rswa_decode(*args(ws=ws - 1)) == INVALID and "workspace" in _err()
    assert lib.rswa_decode(*args(dims=Dims(2, 4, 96, 128, 64))) == UNSUPPORTED
    assert lib.rswa_decode(*args(dims=Dims(2, 4, 128, 0, 64))) == INVALID
    assert lib.rswa_decode(*args(dims=Dims(2, 0, 128, 128, 64))) == INVALID


def test_srswa_validation():
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 64)
    ws = lib.rswa_workspace_bytes(ctypes.byref(d), 2)
    base = [ctypes.byref(d), A, A, A, A, A, A, 16, A, A, A, A, ctypes.c_float(0.088), A, None, A, ctypes.c_size_t(ws),
            None]
    bad_topk = list(base)
    bad_topk[7] = 0
    assert lib.srswa_decode(*bad_topk) == INVALID and "topk" in _err()
    bad_topk[7] = 33
    assert lib.srswa_decode(*bad_topk) == INVALID
    no_idx = list(base)
    no_idx[5] = None
    assert lib.srswa_decode(*no_idx) == INVALID and "blk_idx" in _err()


def test_route_validation():
    lib = rswa.load()
    d = Dims(2, 1, 128, 1, 32 * 8193)
    call = lambda dims, topk=16, probs=None, ws=256: lib.srswa_route(
        ctypes.byref(dims), A, A, A, ctypes.c_float(1.0), topk, A, A2, probs, None, A, ctypes.c_size_t(ws), None)
    assert call(d) == UNSUPPORTED and "limit" in _err()
    d = Dims(2, 1, 128, 1, 1024)
    assert call(d, topk=0) == INVALID
    assert call(d, probs=MIS) == INVALID
    assert call(d, ws=8) == INVALID


def test_append_and_pool_validation():
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 0)
    assert lib.rswa_append(ctypes.byref(d), A, A, None, A, A, A, None, None, None) == INVALID
    assert lib.rswa_append(ctypes.byref(d), A, A, A, A, None, A, None, None, None) == INVALID
    assert lib.rswa_append(None, A, A, A, A, A, A, None, None, None) == INVALID
    assert lib.srswa_index_pool(ctypes.byref(Dims(2, 1, 128, 1, 64)), None, A, A, None) == INVALID


def test_python_binding_rejects_cpu_tensors():
    import torch
    t = torch.zeros((1, 1, 4, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        rswa.rswa_append(t, t, t[:, :, 0], t[:, :, 0], torch.zeros(1, dtype=torch.int32),
                         torch.zeros(1, dtype=torch.int32))


def test_fp8_entry_points_validation():
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 64)
    st = ctypes.c_void_p(0x30000)
    q = [ctypes.byref(d), A, A, A, A, A, A, A, st, None]           # valid: never called as is (it would launch)
    bad = list(q)
    bad[4] = None                                                      # pk8
    assert lib.rswa_quantize_prefix(*bad) == INVALID and "pk8" in _err()
    bad = list(q)
    bad[6] = MIS                                                       # k_scale
    assert lib.rswa_quantize_prefix(*bad) == INVALID and "aligned" in _err()
    ws = lib.rswa_workspace_bytes(ctypes.byref(d), 1)
    dec = [ctypes.byref(d), A, A, A, None, A, A, A, A, A, A, ctypes.c_float(0.088), A, None, A, ctypes.c_size_t(ws),
           None]
    assert lib.rswa_decode_fp8(*dec) == INVALID and "k_scale" in _err()


def test_chunked_prefill_entry_points_validation():
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 64)
    route = lambda T, dims=d: lib.srswa_route_tokens(ctypes.byref(dims), T, A, A, A, ctypes.c_float(1.0), 16, A, A, A,
                                                     ctypes.c_size_t(256), None)
    assert route(0) == INVALID and "T must be" in _err()
    assert route(40000) == UNSUPPORTED and "65535" in _err()
    pf = lambda T=8, k_out=A, ring_k=None, ring_v=None: lib.srswa_prefill(
        ctypes.byref(d), T, A, k_out, A, A, A, A, A, A, 16, ring_k, ring_v, None, None, ctypes.c_float(0.088), A, None,
        A, ctypes.c_size_t(256), None)
    assert pf(T=0) == INVALID and "T must be" in _err()
    assert pf(k_out=MIS) == INVALID and "aligned" in _err()
    assert pf(ring_k=A) == INVALID and "both" in _err()
    assert pf(ring_k=A, ring_v=A2) == INVALID and "wp and fill" in _err()
    assert pf(T=9000) == UNSUPPORTED and "8192" in _err()
    assert pf() == INVALID and "srswa_prefill_workspace_bytes" in _err()      # 256 bytes are too few
    assert lib.srswa_prefill_workspace_bytes(ctypes.byref(d), 8) > 256


def test_fused_step_validation():
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 64)
    ws = lib.rswa_workspace_bytes(ctypes.byref(d), 1)
    call = lambda k_new=A, ws_bytes=ws: lib.rswa_decode_append(
        ctypes.byref(d), A, k_new, A, A, A, A, A, A, A, A, None, ctypes.c_float(0.088), A, None, A,
        ctypes.c_size_t(ws_bytes), None)
    assert call(k_new=None) == INVALID and "k_new" in _err()
    assert call(k_new=MIS) == INVALID and "aligned" in _err()
    assert call(ws_bytes=255) == INVALID and "workspace" in _err()


def test_rope_entry_points_validation():
    lib = rswa.load()
    D64 = ctypes.c_double

    def rope(rows=8, heads=4, head_dim=128, q=A, q_out=A, k=None, k_out=None, tok=A, page=A2, base=1e4, page_mod=2):
        return lib.rswa_rope_page2d(rows, heads, head_dim, q, q_out, k, k_out, tok, page, D64(base), page_mod, None)

    assert rope(rows=-1) == INVALID and "rows" in _err()
    assert rope(heads=0) == INVALID and "heads" in _err()
    assert rope(head_dim=100) == UNSUPPORTED and "head_dim" in _err()
    assert rope(head_dim=272) == UNSUPPORTED
    assert rope(q=None) == INVALID and "q must not be NULL" in _err()
    assert rope(q_out=MIS) == INVALID and "aligned" in _err()
    assert rope(k=A) == INVALID and "both" in _err()
    assert rope(k=MIS, k_out=A) == INVALID and "aligned" in _err()
    assert rope(tok=None) == INVALID and "tok_pos" in _err()
    assert rope(base=0.0) == INVALID and "base" in _err()
    assert rope(base=float("inf")) == INVALID
    assert rope(page_mod=-1) == INVALID and "page_mod" in _err()
    assert rope(rows=0) == 0 and _err() == ""          # nothing to encode: no launch
    assert rope(rows=0, q=None, q_out=None, tok=None, page=None) == 0     # empty tensors have NULL data
    assert rope(rows=0, head_dim=100) == UNSUPPORTED and rope(rows=0, base=-1.0) == INVALID

    d = Dims(2, 4, 128, 128, 0)

    def app(dims=d, q=A, q_out=A, wp=A, page=A2, base=1e4, page_mod=2):
        return lib.rswa_append_rope(ctypes.byref(dims), A, A, A, A, wp, A, None, q, q_out, A, page, D64(base),
                                    page_mod, None, None)

    assert app(dims=Dims(2, 4, 64, 128, 0)) == UNSUPPORTED and "head_dim" in _err()
    assert app(q=None) == INVALID and "q must not be NULL" in _err()
    assert app(q_out=MIS) == INVALID and "aligned" in _err()
    assert app(wp=None) == INVALID and "wp and fill" in _err()
    assert app(page=None) == INVALID and "page" in _err()
    assert app(base=float("nan")) == INVALID and "base" in _err()
    assert app(page_mod=-2) == INVALID and "page_mod" in _err()


def test_missing_library_fails_loudly(tmp_path):
    # no CPU fallback: without the library every call path raises
    import subprocess
    import sys
    env = dict(os.environ, RSWA_LIBRARY=str(tmp_path / "absent" / "librswa.so"))
    code = "import long_context_decode_swa_b200 as r\nr.load()"
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, env=env, cwd=ROOT, timeout=300)
    assert out.returncode != 0 and "not found" in out.stderr


def test_fp8_ring_entry_points_validation():
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 64)
    ws = lib.rswa_workspace_bytes(ctypes.byref(d), 1)

    def dec(ring_k8=A, ring_vscale=A, pk8=A, ws_bytes=ws):
        return lib.rswa_decode_fp8kv(ctypes.byref(d), A, pk8, A, A, A, A, ring_k8, A, A, ring_vscale, A, A,
                                     ctypes.c_float(0.088), A, None, A, ctypes.c_size_t(ws_bytes), None)

    assert dec(ring_k8=None) == INVALID and "ring_k8" in _err()
    assert dec(ring_vscale=MIS) == INVALID and "aligned" in _err()
    assert dec(pk8=None) == INVALID
    assert dec(ws_bytes=16) == INVALID and "workspace" in _err()

    def app(ring_k8=A, k_new=A, wp=A, dims=d):
        return lib.rswa_append_fp8(ctypes.byref(dims), ring_k8, A, A, A, k_new, A, wp, A, None, None, None)

    assert app(ring_k8=None) == INVALID and "ring_k8" in _err()
    assert app(k_new=MIS) == INVALID and "aligned" in _err()
    assert app(wp=None) == INVALID and "wp and fill" in _err()
    assert app(dims=Dims(2, 4, 64, 128, 0)) == UNSUPPORTED


def test_wait_timeout_hook_validation():
    lib = rswa.load()
    assert lib.rswa_test_arm_wait_timeout(-2, 20_000_000) == INVALID and "drop_tile" in _err()
    assert lib.rswa_test_arm_wait_timeout(0, 10) == INVALID and "wait_limit_ns" in _err()
    assert lib.rswa_test_arm_wait_timeout(0, 20_000_000) == 0
    # the armed knob is consumed by the next decode-family call even when that call fails validation
    d = Dims(2, 4, 128, 128, 64)
    assert lib.rswa_decode(ctypes.byref(d), None, A, A, A, A, A, A, A, ctypes.c_float(0.088), A, None, A,
                           ctypes.c_size_t(1 << 20), None) == INVALID


def test_fused_router_entry_points_validation():
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 64 * 32)
    ws = lib.rswa_workspace_bytes(ctypes.byref(d), 5)
    assert ws > lib.rswa_workspace_bytes(ctypes.byref(d), 2)   # the decode plan plus the router's area

    def routed(q_idx=A, kbar=A, topk=16, blk=A, idx_scale=1.0, dims=d):
        return lib.srswa_decode_routed(ctypes.byref(dims), A, q_idx, kbar, ctypes.c_float(idx_scale), topk, A, A, A,
                                       A, A, A, A, ctypes.c_float(0.088), blk, A, None, A, None, A,
                                       ctypes.c_size_t(ws), None)

    assert routed(q_idx=None) == INVALID and "q_idx" in _err()
    assert routed(kbar=MIS) == INVALID and "aligned" in _err()
    assert routed(topk=33) == INVALID and "topk" in _err()
    assert routed(blk=None) == INVALID
    assert routed(idx_scale=float("inf")) == INVALID and "idx_scale" in _err()
    assert routed(dims=Dims(2, 4, 128, 128, 8193 * 32)) == UNSUPPORTED and "limit" in _err()

    def step(k_new=A, slot_out=None):
        return lib.srswa_step(ctypes.byref(d), A, k_new, A, A, A, ctypes.c_float(1.0), 16, A, A, A, A, A, A, A,
                              slot_out, ctypes.c_float(0.088), A, A, None, A, None, A, ctypes.c_size_t(ws), None)

    assert step(k_new=None) == INVALID and "k_new" in _err()


def test_fused_steps_with_encoding_validation():
    from long_context_decode_swa_b200.binding import Rope
    lib = rswa.load()
    d = Dims(2, 4, 128, 128, 64 * 32)
    ws_dec = lib.rswa_workspace_bytes(ctypes.byref(d), 1)
    ws_step = lib.rswa_workspace_bytes(ctypes.byref(d), 5)

    def dec(rope=True, tok=A, page=A2, base=1e4, page_mod=2, k_new=A, ws_bytes=ws_dec):
        r = Rope(tok, page, base, page_mod)
        return lib.rswa_decode_append_rope(ctypes.byref(d), ctypes.byref(r) if rope else None, A, k_new, A, A, A, A,
                                           A, A, A, A, None, ctypes.c_float(0.088), A, None, A,
                                           ctypes.c_size_t(ws_bytes), None)

    assert dec(rope=False) == INVALID and "rope" in _err()
    assert dec(tok=None) == INVALID and "tok_pos" in _err()
    assert dec(page=None) == INVALID and "page" in _err()
    assert dec(base=0.0) == INVALID and "base" in _err()
    assert dec(base=float("nan")) == INVALID and "base" in _err()
    assert dec(page_mod=-1) == INVALID and "page_mod" in _err()
    assert dec(k_new=None) == INVALID and "k_new" in _err()
    assert dec(ws_bytes=255) == INVALID and "workspace" in _err()

    def step(rope=True, tok=A, base=1e4, page_mod=2, q_idx=A, ws_bytes=ws_step):  # the size check needs a GPU
        r = Rope(tok, A2, base, page_mod)
        return lib.srswa_step_rope(ctypes.byref(d), ctypes.byref(r) if rope else None, A, A, A, q_idx, A,
                                   ctypes.c_float(1.0), 16, A, A, A, A, A, A, A, None, ctypes.c_float(0.088), A, A,
                                   None, A, None, A, ctypes.c_size_t(ws_bytes), None)

    assert step(rope=False) == INVALID and "rope" in _err()
    assert step(tok=None) == INVALID and "tok_pos" in _err()
    assert step(base=-3.0) == INVALID and "base" in _err()
    assert step(page_mod=-5) == INVALID and "page_mod" in _err()
    assert step(q_idx=None) == INVALID and "q_idx" in _err()
