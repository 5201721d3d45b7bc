"""GPU parity of ring append + R-SWA split-KV decode against the oracle.

Slots, wp, fill and ring bytes are compared bit-exactly; attention outputs
within max-abs 1e-2 and relative L2 1e-4 (gpu_util); lse within 1e-4.
"""
import numpy as np
import pytest
import torch

from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, DecodeRunner, assert_attention_close, to_np

pytestmark = pytest.mark.gpu


def _run(rswa, case, steps, check_steps, sample=None, tag=""):
    r = DecodeRunner(rswa, case, sample)
    for s in range(steps):
        o_slot = r.step(s)
        np.testing.assert_array_equal(to_np(r.slot), o_slot, err_msg=f"{tag} slot_out step {s}")
        if s in check_steps:
            r.check_ring()
            ref, ref_lse = r.oracle_rswa(s)
            got, got_lse = r.gpu_out()
            assert_attention_close(got, ref, f"{tag} step {s}")
            assert np.abs(got_lse - ref_lse).max() <= LSE_ABS, f"{tag} lse step {s}"
    assert rswa.check_status(r.ws) == 0
    return r


@pytest.mark.parametrize("plen,n,wp0,fill0,steps", [
    ([5, 77, 200], 40, [0, 13, 39], [0, 40, 17], 90),     # ragged prefixes, ring wraps, partial tiles
    ([1, 32, 64], 128, 0, 0, 140),                      # empty ring filling past n
    ([200, 199, 33], 100, None, 100, 30),               # n not a multiple of 32, full ring
])
def test_decode_small_shapes(cuda_lib, plen, n, wp0, fill0, steps):
    case = synth.decode_case(3, 4, 128, plen, 200, n, steps, seed=101, device="cuda", wp0=wp0, fill0=fill0)
    _run(cuda_lib, case, steps, set(range(0, steps, 7)) | {steps - 1}, tag=f"plen={plen} n={n}")


def test_decode_long_pipelines(cuda_lib):
    # 80 x 16 (sequence, head) pairs leave one split per pair, so each CTA streams ~36 tiles
    # through its stage ring (every stage reused many times), with ragged prefix tails
    plen = [1000 - 7 * (b % 5) for b in range(80)]
    case = synth.decode_case(80, 16, 128, plen, 1000, 128, 3, seed=102, device="cuda")
    sample = np.arange(0, 80, 9)
    _run(cuda_lib, case, 3, {0, 1, 2}, sample=sample, tag="long pipelines")


def test_decode_config1_single_sequence(cuda_lib):
    # batch 1, 16 heads, prefix 256 visual + 32 prompt, full 128-slot ring with wp at slot 37, 64 steps
    m = synth.ocr_prefix_len(1)
    case = synth.decode_case(1, 16, 128, m, m, 128, 64, seed=1001, device="cuda", wp0=37, fill0=128)
    _run(cuda_lib, case, 64, set(range(64)), tag="config1")


def test_decode_config2_batched_sampled(cuda_lib):
    # 512 sequences, 10-page prefix (2592 tokens), wp uniform in [0,128), 256 steps; the launch is the
    # benchmark's; the oracle checks 24 sampled sequences at steps 0, 1, 127, 128, 255 and every slot
    m = synth.ocr_prefix_len(10)
    case = synth.decode_case(512, 16, 128, m, m, 128, 256, seed=2001, device="cuda")
    sample = np.sort(np.random.default_rng(5).choice(512, 24, replace=False))
    _run(cuda_lib, case, 256, {0, 1, 127, 128, 255}, sample=sample, tag="config2")


def test_decode_peaked_queries(cuda_lib):
    # queries scaled x4 make the softmax peaked and exercise the running-max rescale
    case = synth.decode_case(4, 16, 128, [700, 333, 1, 64], 700, 128, 8, seed=103, device="cuda", q_std=4.0)
    _run(cuda_lib, case, 8, set(range(8)), tag="peaked")


@pytest.mark.parametrize("n", [1, 2, 256])
def test_decode_edge_ring_sizes(cuda_lib, n):
    case = synth.decode_case(2, 2, 128, [0, 45], 45, n, 2 * n + 3, seed=104, device="cuda", wp0=0, fill0=0)
    _run(cuda_lib, case, 2 * n + 3, {0, 1, n - 1, n, 2 * n + 2}, tag=f"n={n}")


def test_decode_empty_prefix_single_key_is_v_self(cuda_lib):
    case = synth.decode_case(3, 2, 128, 0, 1, 16, 1, seed=105, device="cuda", wp0=[0, 5, 15], fill0=0)
    r = DecodeRunner(cuda_lib, case)
    r.step(0)
    got, _ = r.gpu_out()
    v_self = case.v_new[0].float().cpu().numpy()
    np.testing.assert_array_equal(got, v_self)


def test_decode_many_heads_and_max_prefix(cuda_lib):
    # prefix_len == prefix_cap for one sequence, 64 heads, and a split-KV plan with several splits
    case = synth.decode_case(2, 64, 128, [4096, 1000], 4096, 128, 2, seed=106, device="cuda")
    _run(cuda_lib, case, 2, {0, 1}, tag="H=64")


def test_device_checks_flag_bad_state(cuda_lib):
    rswa = cuda_lib
    case = synth.decode_case(2, 2, 128, [10, 10], 10, 8, 1, seed=107, device="cuda")
    r = DecodeRunner(rswa, case)
    bad_plen = torch.tensor([11, 10], dtype=torch.int32, device="cuda")          # > prefix_cap
    rswa.rswa_decode(case.q[0], case.pk, case.pv, bad_plen, r.ring_k, r.ring_v, r.wp, r.fill, r.out, r.ws)
    assert rswa.check_status(r.ws) & rswa.binding.DEVICE_BAD_PREFIX_LEN
    bad_wp = torch.tensor([8, 0], dtype=torch.int32, device="cuda")              # wp == n
    rswa.rswa_append(r.ring_k, r.ring_v, case.k_new[0], case.v_new[0], bad_wp, r.fill, status=r.ws)
    assert rswa.check_status(r.ws) & rswa.binding.DEVICE_BAD_RING_STATE
    assert bad_wp.tolist() == [8, 1]                                              # seq 0 untouched
    assert rswa.check_status(r.ws) == 0                                           # cleared


def test_workspace_is_reusable_across_calls(cuda_lib):
    # the merging CTA resets the per-(b,h) counters: repeated calls give identical results
    case = synth.decode_case(1, 16, 128, 288, 288, 128, 1, seed=108, device="cuda", wp0=37, fill0=128)
    r = DecodeRunner(cuda_lib, case)
    r.step(0)
    first = r.out.clone()
    for _ in range(3):
        cuda_lib.rswa_decode(case.q[0], case.pk, case.pv, case.prefix_len, r.ring_k, r.ring_v, r.wp, r.fill, r.out,
                             r.ws, scale=case.scale)
        assert torch.equal(r.out, first)
    counters = r.ws[256:256 + 4 * 16].view(torch.int32)
    assert int(counters.abs().sum()) == 0
