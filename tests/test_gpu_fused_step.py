"""GPU parity of the fused decode step (ring append + decode in one launch) against the
oracle's append followed by its decode: slot_out, wp, fill and the ring bit-exact every
step; outputs within max-abs 1e-2 / relative L2 1e-4, lse within 1e-4."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, DecodeRunner, assert_attention_close, to_np

pytestmark = pytest.mark.gpu


class FusedRunner(DecodeRunner):
    def step(self, s: int, sparse=None):
        c = self.c
        if sparse is None:
            self.rswa.rswa_decode_append(c.q[s], c.k_new[s], c.v_new[s], c.pk, c.pv, c.prefix_len, self.ring_k,
                                         self.ring_v, self.wp, self.fill, self.out, self.ws, lse=self.lse,
                                         slot_out=self.slot, scale=c.scale)
        else:
            self.rswa.srswa_decode_append(c.q[s], c.k_new[s], c.v_new[s], c.pk, c.pv, c.prefix_len, sparse[0],
                                          sparse[1], self.ring_k, self.ring_v, self.wp, self.fill, self.out,
                                          self.ws_sparse, lse=self.lse, slot_out=self.slot, scale=c.scale)
        return oracle.append(self.o_ring_k, self.o_ring_v, to_np(c.k_new[s]), to_np(c.v_new[s]), self.o_wp,
                             self.o_fill)


def _run(rswa, case, steps, check, sample=None, tag=""):
    r = FusedRunner(rswa, case, sample)
    for s in range(steps):
        o_slot = r.step(s)
        np.testing.assert_array_equal(to_np(r.slot), o_slot, err_msg=f"{tag} slot_out step {s}")
        np.testing.assert_array_equal(to_np(r.wp), r.o_wp, err_msg=f"{tag} wp step {s}")
        np.testing.assert_array_equal(to_np(r.fill), r.o_fill, err_msg=f"{tag} fill step {s}")
        if s in check:
            r.check_ring()
            ref, ref_lse = r.oracle_rswa(s)
            got, got_lse = r.gpu_out()
            assert_attention_close(got, ref, f"{tag} step {s}")
            assert np.abs(got_lse - ref_lse).max() <= LSE_ABS, f"{tag} lse step {s}"
    assert rswa.check_status(r.ws) == 0
    assert int(r.ws[128:132].view(torch.int32).item()) == 0          # the completion counter is rearmed
    return r


@pytest.mark.parametrize("plen,n,wp0,fill0,steps", [
    ([5, 77, 200], 40, [0, 13, 39], [0, 40, 17], 90),     # empty / full / partial rings that wrap
    ([1, 32, 64], 128, 0, 0, 140),                      # empty ring filling past n
    ([200, 199, 33], 100, None, 100, 30),               # n not a multiple of 32, full ring
])
def test_fused_step_small_shapes(cuda_lib, plen, n, wp0, fill0, steps):
    case = synth.decode_case(3, 4, 128, plen, 200, n, steps, seed=401, device="cuda", wp0=wp0, fill0=fill0)
    _run(cuda_lib, case, steps, set(range(0, steps, 7)) | {steps - 1}, tag=f"fused plen={plen} n={n}")


def test_fused_step_split_kv(cuda_lib):
    # two long sequences: several splits per (sequence, head); this step's token is in the last one
    case = synth.decode_case(2, 8, 128, [9000, 4097], 9000, 128, 4, seed=402, device="cuda", wp0=[5, 127])
    _run(cuda_lib, case, 4, {0, 1, 2, 3}, tag="fused split-kv")


def test_fused_step_single_sequence_and_batched(cuda_lib):
    m = synth.ocr_prefix_len(1)
    case = synth.decode_case(1, 16, 128, m, m, 128, 40, seed=403, device="cuda", wp0=37, fill0=128)
    _run(cuda_lib, case, 40, set(range(0, 40, 3)), tag="fused single")
    m = synth.ocr_prefix_len(10)
    case = synth.decode_case(512, 16, 128, m, m, 128, 3, seed=404, device="cuda")
    sample = np.sort(np.random.default_rng(7).choice(512, 12, replace=False))
    _run(cuda_lib, case, 3, {0, 1, 2}, sample=sample, tag="fused batched")


def test_fused_srswa_step(cuda_lib):
    plen = [32 * 48, 32 * 40 + 9, 32 * 17]
    case = synth.decode_case(3, 16, 128, plen, 32 * 48, 128, 4, seed=405, device="cuda", fill0=[128, 60, 0])
    r = FusedRunner(cuda_lib, case)
    rng = np.random.default_rng(10)
    for s in range(4):
        blk = np.stack([rng.permutation((m + 31) // 32)[:16] for m in plen]).astype(np.int32)
        logp = np.log(rng.dirichlet(np.ones(16), size=3)).astype(np.float32)
        blk[1, 4] = -1
        o_slot = r.step(s, sparse=(torch.from_numpy(blk).cuda(), torch.from_numpy(logp).cuda()))
        np.testing.assert_array_equal(to_np(r.slot), o_slot)
        r.check_ring()
        ref, ref_lse = r.oracle_srswa(s, blk, logp.astype(np.float64))
        got, got_lse = r.gpu_out()
        assert_attention_close(got, ref, f"fused srswa step {s}")
        assert np.abs(got_lse - ref_lse).max() <= LSE_ABS
    assert cuda_lib.check_status(r.ws_sparse) == 0


def test_fused_step_bad_ring_state_is_flagged_and_left_alone(cuda_lib):
    case = synth.decode_case(2, 4, 128, [64, 64], 64, 16, 1, seed=406, device="cuda", wp0=[3, 3], fill0=[16, 16])
    r = FusedRunner(cuda_lib, case)
    r.wp[1] = 99                                                      # out of range
    r.step(0)
    assert int(r.wp[1]) == 99 and int(r.fill[1]) == 16              # untouched
    assert int(r.wp[0]) == 4 and int(r.fill[0]) == 16                # the good sequence advanced
    st = cuda_lib.check_status(r.ws)
    assert st & cuda_lib.binding.DEVICE_BAD_RING_STATE
