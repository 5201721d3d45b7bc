"""GPU parity of the FP8 (E4M3) prefix path against the oracle.

- rswa_quantize_prefix: codes and block scales bit-exact against the oracle's
  quantiser (both take amax / 448 and x / scale in fp32, round to nearest even).
- rswa_decode_fp8 / srswa_decode_fp8: the prefix codes and scales come from
  the oracle's quantiser on the CPU, or (large cases) are drawn directly by the
  seeded generator; no input comes from the CUDA path. Both sides read the same
  codes and scales; outputs within the decode tolerances (max-abs 1e-2,
  relative L2 1e-4), lse within 1e-4.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, DecodeRunner, assert_attention_close, to_np

pytestmark = pytest.mark.gpu


def _scaled_prefix(B, H, cap, seed):
    """bf16 prefix with row-dependent magnitudes (block scales spread over ~e^+-3)."""
    g = torch.Generator(device="cuda").manual_seed(seed)
    x = torch.randn((B, H, cap, 128), generator=g, device="cuda")
    mag = torch.exp(torch.randn((B, H, cap, 1), generator=g, device="cuda"))
    return (x * mag).bfloat16()


@pytest.mark.parametrize("plen,cap", [([200, 64, 0], 224), ([31, 1, 224], 224), ([2592] * 2, 2592)])
def test_quantize_prefix_bit_exact(cuda_lib, plen, cap):
    B, H = len(plen), 4
    pk = _scaled_prefix(B, H, cap, 7)
    pv = _scaled_prefix(B, H, cap, 8)
    pl = torch.tensor(plen, dtype=torch.int32, device="cuda")
    k8 = torch.zeros((B, H, cap, 128), dtype=torch.uint8, device="cuda")
    v8 = torch.zeros_like(k8)
    ks = torch.zeros((B, H, (cap + 31) // 32), dtype=torch.float32, device="cuda")
    vs = torch.zeros_like(ks)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    cuda_lib.rswa_quantize_prefix(pk, pv, pl, k8, v8, ks, vs, status=ws)
    assert cuda_lib.check_status(ws) == 0
    for x, codes, scales in ((pk, k8, ks), (pv, v8, vs)):
        o_codes, o_scales = oracle.quantize_prefix(to_np(x), np.array(plen, np.int32))
        np.testing.assert_array_equal(to_np(scales), o_scales)
        np.testing.assert_array_equal(to_np(codes), o_codes)


class FP8Runner(DecodeRunner):
    """DecodeRunner whose prefix is read as E4M3 codes and block scales: the oracle's quantisation
    of the case's bf16 prefix (quantised=True), or codes and scales drawn directly (synth.fp8_prefix)."""

    def __init__(self, rswa, case, sample=None, quantised=True, seed=0):
        super().__init__(rswa, case, sample)
        sm = self.sample
        if quantised:
            plen = to_np(case.prefix_len)
            k8, ks = oracle.quantize_prefix(to_np(case.pk), plen)
            v8, vs = oracle.quantize_prefix(to_np(case.pv), plen)
            self.k8, self.v8 = torch.from_numpy(k8).cuda(), torch.from_numpy(v8).cuda()
            self.ks, self.vs = torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda()
        else:
            B, H, cap, _ = case.pk.shape
            self.k8, self.v8, self.ks, self.vs = synth.fp8_prefix(B, H, cap, seed, device="cuda")
        sel = torch.as_tensor(sm, device="cuda")
        self.o_k8, self.o_v8 = to_np(self.k8.index_select(0, sel)), to_np(self.v8.index_select(0, sel))
        self.o_ks, self.o_vs = to_np(self.ks.index_select(0, sel)), to_np(self.vs.index_select(0, sel))

    def step(self, s: int, sparse=None):
        c = self.c
        self.rswa.rswa_append(self.ring_k, self.ring_v, c.k_new[s], c.v_new[s], self.wp, self.fill,
                              slot_out=self.slot, status=self.ws)
        if sparse is None:
            self.rswa.rswa_decode_fp8(c.q[s], self.k8, self.v8, self.ks, self.vs, c.prefix_len, self.ring_k,
                                      self.ring_v, self.wp, self.fill, self.out, self.ws, lse=self.lse, scale=c.scale)
        else:
            self.rswa.srswa_decode_fp8(c.q[s], self.k8, self.v8, self.ks, self.vs, c.prefix_len, sparse[0],
                                       sparse[1], self.ring_k, self.ring_v, self.wp, self.fill, self.out,
                                       self.ws_sparse, lse=self.lse, scale=c.scale)
        return oracle.append(self.o_ring_k, self.o_ring_v, to_np(c.k_new[s]), to_np(c.v_new[s]), self.o_wp,
                             self.o_fill)

    def _ring_state(self):
        sm = self.sample
        return (np.ascontiguousarray(self.o_ring_k[sm]), np.ascontiguousarray(self.o_ring_v[sm]),
                self.o_wp[sm].copy(), self.o_fill[sm].copy(), self.c.scale)

    def oracle_rswa(self, s: int):
        return oracle.rswa_decode_fp8(to_np(self.c.q[s])[self.sample], self.o_k8, self.o_v8, self.o_ks, self.o_vs,
                                      self.o_plen, *self._ring_state())

    def oracle_srswa(self, s: int, blk_idx, blk_logp):
        sm = self.sample
        return oracle.srswa_decode_fp8(to_np(self.c.q[s])[sm], self.o_k8, self.o_v8, self.o_ks, self.o_vs,
                                       self.o_plen, np.ascontiguousarray(blk_idx[sm]),
                                       np.ascontiguousarray(blk_logp[sm]), *self._ring_state())


def _run(rswa, case, steps, check, sample=None, tag="", quantised=True):
    r = FP8Runner(rswa, case, sample, quantised=quantised, seed=int(case.prefix_len.sum().item()) % 1000 + 7)
    for s in range(steps):
        r.step(s)
        if s in check:
            ref, ref_lse = r.oracle_rswa(s)
            got, got_lse = r.gpu_out()
            assert_attention_close(got, ref, f"{tag} step {s}")
            assert np.abs(got_lse - ref_lse).max() <= LSE_ABS, f"{tag} lse step {s}"
    assert rswa.check_status(r.ws) == 0


@pytest.mark.parametrize("plen,n,wp0,fill0,steps", [
    ([5, 77, 200], 40, [0, 13, 39], [0, 40, 17], 45),     # ragged prefixes and partial blocks, ring wraps
    ([200, 199, 33], 100, None, 100, 12),                # n not a multiple of 32, full ring
])
def test_decode_fp8_small_shapes(cuda_lib, plen, n, wp0, fill0, steps):
    case = synth.decode_case(3, 4, 128, plen, 200, n, steps, seed=301, device="cuda", wp0=wp0, fill0=fill0)
    _run(cuda_lib, case, steps, set(range(0, steps, 5)) | {steps - 1}, tag=f"fp8 plen={plen} n={n}")


def test_decode_fp8_split_kv_and_long_pipelines(cuda_lib):
    # one long sequence (many splits per (b, h)) next to a batch of ragged ones
    case = synth.decode_case(2, 16, 128, [9000, 4097], 9000, 128, 2, seed=302, device="cuda")
    _run(cuda_lib, case, 2, {0, 1}, tag="fp8 split-kv", quantised=False)
    plen = [1000 - 7 * (b % 5) for b in range(80)]
    case = synth.decode_case(80, 16, 128, plen, 1000, 128, 2, seed=303, device="cuda")
    _run(cuda_lib, case, 2, {0, 1}, sample=np.arange(0, 80, 9), tag="fp8 long pipelines", quantised=False)


def test_decode_fp8_batched_workload_sampled(cuda_lib):
    # the batched workload's shape: 512 sequences, 10-page prefix, full ring, wp uniform
    m = synth.ocr_prefix_len(10)
    case = synth.decode_case(512, 16, 128, m, m, 128, 2, seed=2006, device="cuda")
    sample = np.sort(np.random.default_rng(6).choice(512, 12, replace=False))
    _run(cuda_lib, case, 2, {0, 1}, sample=sample, tag="fp8 batched", quantised=False)


def test_decode_fp8_peaked_queries(cuda_lib):
    case = synth.decode_case(4, 16, 128, [700, 333, 1, 64], 700, 128, 4, seed=304, device="cuda", q_std=4.0)
    _run(cuda_lib, case, 4, set(range(4)), tag="fp8 peaked")


def test_srswa_decode_fp8_given_route(cuda_lib):
    plen = [32 * 48, 32 * 40 + 9, 32 * 17]
    cap = 32 * 48
    case = synth.decode_case(3, 16, 128, plen, cap, 128, 3, seed=305, device="cuda")
    r = FP8Runner(cuda_lib, case)
    rng = np.random.default_rng(9)
    for s in range(3):
        blk = np.stack([rng.permutation((m + 31) // 32)[:16] for m in plen]).astype(np.int32)
        blk[1, 5] = -1                                                    # a skipped entry
        logp = np.log(rng.dirichlet(np.ones(16), size=3)).astype(np.float32)
        logp[2, 3] = -np.inf                                              # a zero-probability entry
        r.step(s, sparse=(torch.from_numpy(blk).cuda(), torch.from_numpy(logp).cuda()))
        ref, ref_lse = r.oracle_srswa(s, blk, logp.astype(np.float64))
        got, got_lse = r.gpu_out()
        assert_attention_close(got, ref, f"fp8 srswa step {s}")
        assert np.abs(got_lse - ref_lse).max() <= LSE_ABS
    assert cuda_lib.check_status(r.ws_sparse) == 0
