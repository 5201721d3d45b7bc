"""The decode kernels' bounded-wait path, exercised on the GPU without a fault.

rswa_test_arm_wait_timeout makes the next decode call's CTA 0 skip one tile's copy while
its warp still waits on that tile's shared-memory stage: nothing ever fills the stage, the
bounded wait runs out after the short limit given, the kernel sets
RSWA_DEVICE_WAIT_TIMEOUT, lets its other copies in flight land and ends, and the call
returns with the context usable. The checks: the status bit is set, the stream finishes
within a small multiple of the limit, rswa_check_status returns the workspace to its
zero-filled state (split-KV plans leave completion counters behind when a CTA gives up),
and the next normal call on the same workspace matches the oracle.
"""
import time

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, assert_attention_close, to_np

pytestmark = pytest.mark.gpu

LIMIT_NS = 20_000_000  # 20 ms


def _decode(rswa, c, ring_k, ring_v, wp, fill, out, lse, ws):
    rswa.rswa_decode(c.q[0], c.pk, c.pv, c.prefix_len, ring_k, ring_v, wp, fill, out, ws, lse=lse, scale=c.scale)


@pytest.mark.parametrize("B,H,plen,drop", [
    (2, 4, [300, 77], 0),      # one split per (sequence, head): CTA 0's first tile
    (8, 16, [4000] * 8, 6),    # two splits per (sequence, head) on 148 SMs (completion counters in
                               # use), 64 tiles per item: warp 0's second tile
])
def test_wait_timeout_sets_status_and_recovers(cuda_lib, B, H, plen, drop):
    rswa = cuda_lib
    c = synth.decode_case(B, H, 128, plen, max(plen), 40, 1, seed=321 + B, device="cuda", fill0=40)
    dims = rswa.dims_of(c.pk, c.ring_k)
    ws = rswa.new_workspace(dims, rswa.OP_DECODE)
    out = torch.empty((B, H, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")

    rswa.test_arm_wait_timeout(drop, LIMIT_NS)
    t0 = time.perf_counter()
    _decode(rswa, c, c.ring_k, c.ring_v, c.wp, c.fill, out, lse, ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    status = rswa.check_status(ws)
    assert status & rswa.binding.DEVICE_WAIT_TIMEOUT, f"status 0x{status:x}"
    assert elapsed < 2.0, f"the call took {elapsed:.2f} s with a {LIMIT_NS / 1e6:.0f} ms wait limit"
    assert int(ws.count_nonzero()) == 0, "check_status left the workspace dirty after a timeout"

    # the knob applied to that call only: the next call on the same workspace is normal
    _decode(rswa, c, c.ring_k, c.ring_v, c.wp, c.fill, out, lse, ws)
    assert rswa.check_status(ws) == 0
    ref, ref_lse = oracle.rswa_decode(to_np(c.q[0]), to_np(c.pk), to_np(c.pv), to_np(c.prefix_len), to_np(c.ring_k),
                                      to_np(c.ring_v), to_np(c.wp), to_np(c.fill), c.scale)
    assert_attention_close(to_np(out), ref, "decode after a timed-out call")
    assert np.abs(to_np(lse) - ref_lse).max() <= LSE_ABS


def test_arm_rejects_bad_values(cuda_lib):
    with pytest.raises(cuda_lib.RswaError):
        cuda_lib.test_arm_wait_timeout(-2, LIMIT_NS)
    with pytest.raises(cuda_lib.RswaError):
        cuda_lib.test_arm_wait_timeout(0, 10)
