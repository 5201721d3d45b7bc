"""GPU parity of the FP8 ring (rswa_append_fp8, rswa_decode_fp8kv, srswa_decode_fp8kv)
against the oracle (oracle.append_fp8, rswa_decode_fp8kv, srswa_decode_fp8kv).

- rswa_append_fp8: every step, the written rows' codes and scales bit-exact against the
  oracle's per-row quantiser (both take amax / 448 and x / scale in fp32, round to nearest
  even, saturate), the untouched rows unchanged, slot_out / wp / fill exact.
- decodes: the FP8 prefix comes from the oracle's quantiser; the ring from the steps above
  (so the GPU ring bytes that the decode reads were first checked equal to the oracle's);
  outputs within the decode tolerances (max-abs 1e-2, relative L2 1e-4), lse within 1e-4,
  with empty, partly filled and wrapped rings and ragged prefixes.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, assert_attention_close, to_np

pytestmark = pytest.mark.gpu


class Ring8Run:
    def __init__(self, rswa, case, sparse):
        self.rswa, self.c, self.sparse = rswa, case, sparse
        B, H, cap, D = case.pk.shape
        n = case.ring_k.shape[2]
        plen = to_np(case.prefix_len)
        k8, ks = oracle.quantize_prefix(to_np(case.pk), plen)
        v8, vs = oracle.quantize_prefix(to_np(case.pv), plen)
        self.o_pre = (k8, v8, ks, vs)
        self.pre = tuple(torch.from_numpy(a).cuda() for a in self.o_pre)
        self.ring = rswa.fp8_ring_buffers((B, H, n, D))
        self.o_ring = oracle.fp8_ring(B, H, n, D)
        self.wp, self.fill = case.wp.clone(), case.fill.clone()      # an empty ring (fill0 = 0)
        self.o_wp, self.o_fill = to_np(case.wp).copy(), to_np(case.fill).copy()
        self.dims = rswa.dims_of(case.pk, case.ring_k)
        self.ws = rswa.new_workspace(self.dims, rswa.OP_SRSWA_DECODE if sparse else rswa.OP_DECODE)
        self.out = torch.empty((B, H, D), dtype=torch.float32, device="cuda")
        self.lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
        self.slot = torch.empty(B, dtype=torch.int32, device="cuda")

    def step(self, s, routes=None):
        c, r = self.c, self.rswa
        r.rswa_append_fp8(*self.ring, c.k_new[s], c.v_new[s], self.wp, self.fill, slot_out=self.slot, status=self.ws)
        o_slot = oracle.append_fp8(*self.o_ring, to_np(c.k_new[s]), to_np(c.v_new[s]), self.o_wp, self.o_fill)
        np.testing.assert_array_equal(to_np(self.slot), o_slot)
        np.testing.assert_array_equal(to_np(self.wp), self.o_wp)
        np.testing.assert_array_equal(to_np(self.fill), self.o_fill)
        for got, want in zip(self.ring, self.o_ring):   # whole rings: written rows and untouched rows
            np.testing.assert_array_equal(to_np(got), want)
        if routes is None:
            r.rswa_decode_fp8kv(c.q[s], *self.pre, c.prefix_len, *self.ring, self.wp, self.fill, self.out, self.ws,
                                lse=self.lse, scale=c.scale)
            ref, ref_lse = oracle.rswa_decode_fp8kv(to_np(c.q[s]), *self.o_pre, to_np(c.prefix_len), *self.o_ring,
                                                    self.o_wp, self.o_fill, c.scale)
        else:
            blk, logp = routes
            r.srswa_decode_fp8kv(c.q[s], *self.pre, c.prefix_len, torch.from_numpy(blk).cuda(),
                                 torch.from_numpy(logp).cuda(), *self.ring, self.wp, self.fill, self.out, self.ws,
                                 lse=self.lse, scale=c.scale)
            ref, ref_lse = oracle.srswa_decode_fp8kv(to_np(c.q[s]), *self.o_pre, to_np(c.prefix_len), blk,
                                                     logp.astype(np.float64), *self.o_ring, self.o_wp, self.o_fill,
                                                     c.scale)
        assert_attention_close(to_np(self.out), ref, f"fp8 ring step {s}")
        assert np.abs(to_np(self.lse) - ref_lse).max() <= LSE_ABS


@pytest.mark.parametrize("plen,n,wp0,steps", [
    ([5, 77, 200], 40, [0, 13, 39], 50),      # rings that fill and wrap, ragged prefixes
    ([2592, 1000], 128, [3, 127], 6),         # the batched shape's prefix, a 128-slot ring
])
def test_rswa_fp8_ring_steps(cuda_lib, plen, n, wp0, steps):
    cap = max(plen)
    case = synth.decode_case(len(plen), 4, 128, plen, cap, n, steps, seed=970 + n, device="cuda", wp0=wp0, fill0=0)
    run = Ring8Run(cuda_lib, case, sparse=False)
    for s in range(steps):
        run.step(s)
    assert cuda_lib.check_status(run.ws) == 0


def test_srswa_fp8_ring_steps(cuda_lib):
    plen = [32 * 48, 32 * 40 + 9, 32 * 17]
    case = synth.decode_case(3, 16, 128, plen, 32 * 48, 128, 8, seed=975, device="cuda", wp0=[0, 64, 127], fill0=0)
    run = Ring8Run(cuda_lib, case, sparse=True)
    rng = np.random.default_rng(976)
    for s in range(8):
        blk = np.stack([rng.permutation((m + 31) // 32)[:16] for m in plen]).astype(np.int32)
        logp = np.log(rng.dirichlet(np.ones(16), 3)).astype(np.float32)
        run.step(s, routes=(blk, logp))
    assert cuda_lib.check_status(run.ws) == 0
