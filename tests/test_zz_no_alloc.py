"""rswa_decode_noalloc: R-SWA decode for callers that cannot allocate.

Some callers cannot call cudaMalloc (allocator-free serving loops, plugins
that only receive raw pointers from an engine that owns every allocation).
rswa_decode_noalloc takes its split-KV scratch from static device memory in
the library instead of a caller workspace. These tests call it through the C
ABI and check it against rswa_decode (same tolerance as the other decode
parity tests) on two calls in a row: with several split-KV partials per
(sequence, head), with one split and many pairs, and with one split and counters
only; on the smallest case also directly against the oracle. The file is named
to be collected last; it passes alone in a fresh process and after the other tests.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from long_context_decode_swa_b200.binding import Dims
from tests.gpu_util import ATTN_MAX_ABS, ATTN_REL_L2, LSE_ABS, assert_attention_close, to_np

UNSUPPORTED = 2


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, c, ring_k, ring_v, wp, fill, out, lse, status):
    B, H, cap, D = c.pk.shape
    dims = Dims(B, H, D, ring_k.shape[2], cap)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.rswa_decode_noalloc(ctypes.byref(dims), _p(c.q[0]), _p(c.pk), _p(c.pv), _p(c.prefix_len), _p(ring_k),
                                   _p(ring_v), _p(wp), _p(fill), ctypes.c_float(c.scale), _p(out), _p(lse),
                                   _p(status), stream)


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,plen,cap", [
    (2, 16, [1000, 613], 1000),     # few (sequence, head) pairs: many split-KV partials in the scratch
    (112, 16, [700] * 112, 700),    # 1792 pairs: a single split, as rswa_decode plans it
    (512, 16, [700] * 512, 700),    # enough pairs for one split: counters only
])
def test_noalloc_matches_rswa_decode_twice(cuda_lib, B, H, plen, cap):
    rswa = cuda_lib
    lib = rswa.load()
    c = synth.decode_case(B, H, 128, plen, cap, 128, 1, seed=4242, device="cuda")
    ring_k, ring_v, wp, fill = c.ring_k.clone(), c.ring_v.clone(), c.wp.clone(), c.fill.clone()
    rswa.rswa_append(ring_k, ring_v, c.k_new[0], c.v_new[0], wp, fill)
    ref_out = torch.empty((B, H, 128), dtype=torch.float32, device="cuda")
    ref_lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    ws = rswa.new_workspace(rswa.dims_of(c.pk, c.ring_k), rswa.OP_DECODE)
    rswa.rswa_decode(c.q[0], c.pk, c.pv, c.prefix_len, ring_k, ring_v, wp, fill, ref_out, ws, lse=ref_lse,
                     scale=c.scale)
    # at these shapes rswa_decode's own plan fits the 4 MiB static scratch, so both calls run the same
    # split plan (the budget only binds for very long prefixes over few (sequence, head) pairs, e.g.
    # 149 sequences x 1 head x 2^20 tokens, beyond a test's memory)
    assert lib.rswa_workspace_bytes(ctypes.byref(Dims(B, H, 128, 128, cap)), 1) <= (4 << 20)
    status = torch.full((4,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full((B, H, 128), float("nan"), dtype=torch.float32, device="cuda")
        lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        code = _noalloc(lib, c, ring_k, ring_v, wp, fill, out, lse, status)
        assert code == 0, lib.rswa_last_error().decode()
        torch.cuda.synchronize()
        assert int(status[0]) == 0, f"call {call}: device status 0x{int(status[0]):x}"
        assert_attention_close(out.cpu().numpy(), ref_out.cpu().numpy(), f"noalloc call {call}",
                               rel_l2=ATTN_REL_L2, max_abs=ATTN_MAX_ABS)
        assert np.abs(lse.cpu().numpy() - ref_lse.cpu().numpy()).max() <= LSE_ABS
        if B == 2:  # the smallest case also against the oracle itself
            o_ref, o_lse = oracle.rswa_decode(to_np(c.q[0]), to_np(c.pk), to_np(c.pv), to_np(c.prefix_len),
                                              to_np(ring_k), to_np(ring_v), to_np(wp), to_np(fill), c.scale)
            assert_attention_close(out.cpu().numpy(), o_ref, f"noalloc call {call} vs the oracle")
            assert np.abs(lse.cpu().numpy() - o_lse).max() <= LSE_ABS
    assert rswa.check_status(ws) == 0


@pytest.mark.gpu
def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_lib):
    lib = cuda_lib.load()
    # 65535 x 128 (sequence, head) completion counters alone need 32 MiB > 4 MiB, even with one split
    dims = Dims(65535, 128, 128, 128, 64)
    x = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = _p(x)
    code = lib.rswa_decode_noalloc(ctypes.byref(dims), p, p, p, p, p, p, p, p, ctypes.c_float(0.088), p, None, None,
                                   None)
    assert code == UNSUPPORTED
    assert "static scratch" in lib.rswa_last_error().decode()
