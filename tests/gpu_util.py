"""Shared helpers of the GPU parity tests: tolerances and the step runner
that drives the CUDA library and the oracle over the same seeded inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from long_context_decode_swa_b200 import synth

# Attention outputs (bf16 in, fp32 accumulate): the max-abs bound is the one
# stated for the method; the relative-L2 bound is tighter, because outputs of
# softmax averages over thousands of N(0,1) rows are small (|o| ~ 0.02).
ATTN_MAX_ABS = 1e-2
ATTN_REL_L2 = 1e-4
LSE_ABS = 1e-4
ROUTER_P_ABS = 1e-5


def assert_attention_close(got: np.ndarray, ref: np.ndarray, what: str, rel_l2: float = ATTN_REL_L2,
                           max_abs: float = ATTN_MAX_ABS):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref).max()
    rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
    assert err <= max_abs, f"{what}: max abs error {err:.3e} > {max_abs}"
    assert rel <= rel_l2, f"{what}: relative L2 error {rel:.3e} > {rel_l2}"


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return synth.to_u16(t)
    return t.detach().cpu().numpy()


class DecodeRunner:
    """Runs rswa_append + (rswa_decode | srswa_decode) steps on the GPU, and the
    oracle's ring append for every sequence plus its decode on a sample."""

    def __init__(self, rswa, case: synth.DecodeCase, sample=None):
        self.rswa = rswa
        self.c = case
        B = case.pk.shape[0]
        self.sample = np.arange(B) if sample is None else np.asarray(sample)
        self.ring_k = case.ring_k.clone()
        self.ring_v = case.ring_v.clone()
        self.wp = case.wp.clone()
        self.fill = case.fill.clone()
        self.dims = rswa.dims_of(case.pk, case.ring_k)
        self.ws = rswa.new_workspace(self.dims, rswa.OP_DECODE)
        self.ws_sparse = rswa.new_workspace(self.dims, rswa.OP_SRSWA_DECODE)
        self.out = torch.empty(case.q.shape[1:], dtype=torch.float32, device="cuda")
        self.lse = torch.empty(case.q.shape[1:3], dtype=torch.float32, device="cuda")
        self.slot = torch.empty(B, dtype=torch.int32, device="cuda")
        # oracle state (host)
        self.o_ring_k = to_np(case.ring_k).copy()
        self.o_ring_v = to_np(case.ring_v).copy()
        self.o_wp = to_np(case.wp).copy()
        self.o_fill = to_np(case.fill).copy()
        sel = torch.as_tensor(self.sample, device=case.pk.device)
        self.o_pk = to_np(case.pk.index_select(0, sel))
        self.o_pv = to_np(case.pv.index_select(0, sel))
        self.o_plen = to_np(case.prefix_len)[self.sample].copy()

    def step(self, s: int, sparse=None):
        """One GPU step; sparse = (blk_idx, blk_logp) tensors for SR-SWA."""
        c = self.c
        self.rswa.rswa_append(self.ring_k, self.ring_v, c.k_new[s], c.v_new[s], self.wp, self.fill,
                              slot_out=self.slot, status=self.ws)
        if sparse is None:
            self.rswa.rswa_decode(c.q[s], c.pk, c.pv, c.prefix_len, self.ring_k, self.ring_v, self.wp, self.fill,
                                  self.out, self.ws, lse=self.lse, scale=c.scale)
        else:
            self.rswa.srswa_decode(c.q[s], c.pk, c.pv, c.prefix_len, sparse[0], sparse[1], self.ring_k, self.ring_v,
                                   self.wp, self.fill, self.out, self.ws_sparse, lse=self.lse, scale=c.scale)
        o_slot = oracle.append(self.o_ring_k, self.o_ring_v, to_np(c.k_new[s]), to_np(c.v_new[s]), self.o_wp,
                               self.o_fill)
        return o_slot

    def oracle_rswa(self, s: int):
        sm = self.sample
        return oracle.rswa_decode(to_np(self.c.q[s])[sm], self.o_pk, self.o_pv, self.o_plen,
                                  np.ascontiguousarray(self.o_ring_k[sm]), np.ascontiguousarray(self.o_ring_v[sm]),
                                  self.o_wp[sm].copy(), self.o_fill[sm].copy(), self.c.scale)

    def oracle_srswa(self, s: int, blk_idx: np.ndarray, blk_logp: np.ndarray):
        sm = self.sample
        return oracle.srswa_decode(to_np(self.c.q[s])[sm], self.o_pk, self.o_pv, self.o_plen,
                                   np.ascontiguousarray(blk_idx[sm]), np.ascontiguousarray(blk_logp[sm]),
                                   np.ascontiguousarray(self.o_ring_k[sm]), np.ascontiguousarray(self.o_ring_v[sm]),
                                   self.o_wp[sm].copy(), self.o_fill[sm].copy(), self.c.scale)

    def check_ring(self):
        sm = self.sample
        np.testing.assert_array_equal(to_np(self.wp), self.o_wp)
        np.testing.assert_array_equal(to_np(self.fill), self.o_fill)
        sel = torch.as_tensor(sm, device="cuda")
        np.testing.assert_array_equal(to_np(self.ring_k.index_select(0, sel)), self.o_ring_k[sm])
        np.testing.assert_array_equal(to_np(self.ring_v.index_select(0, sel)), self.o_ring_v[sm])

    def gpu_out(self):
        sm = self.sample
        return to_np(self.out)[sm], to_np(self.lse)[sm]
