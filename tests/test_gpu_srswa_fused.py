"""GPU parity of the SR-SWA decode with the router fused into the gathered-block attention
(srswa_decode_routed) and of the whole fused step (srswa_step: ring append + router +
attention in one launch) against the oracle's srswa_route / srswa_decode / append.

Selected block indices bit-exact on planted inputs (score gaps >= 0.04, asserted >= 1e-3 on
the oracle's scores); tau and the selected blocks' probabilities within 1e-5; attention
outputs within max-abs 1e-2 and relative L2 1e-4; ring bytes, wp, fill and slot_out bit-exact.
On random scores (many entmax candidates, or fewer candidates than topk) the unique parts
are compared, as for srswa_route.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, ROUTER_P_ABS, assert_attention_close, to_np

pytestmark = pytest.mark.gpu


class Fused:
    """Device state of a fused SR-SWA run and the oracle's state of the same sequences."""

    def __init__(self, rswa, c, kbar, topk=16, sample=None):
        self.rswa, self.c, self.kbar, self.topk = rswa, c, kbar, topk
        B, H, cap, D = c.pk.shape
        self.sample = np.arange(B) if sample is None else np.asarray(sample)
        self.ring_k, self.ring_v = c.ring_k.clone(), c.ring_v.clone()
        self.wp, self.fill = c.wp.clone(), c.fill.clone()
        self.dims = rswa.dims_of(c.pk, c.ring_k)
        self.ws = rswa.new_workspace(self.dims, rswa.OP_SRSWA_ROUTED)
        self.blk = torch.full((B, topk), -7, dtype=torch.int32, device="cuda")
        self.logp = torch.zeros((B, topk), dtype=torch.float32, device="cuda")
        self.tau = torch.zeros((B,), dtype=torch.float32, device="cuda")
        self.out = torch.empty((B, H, D), dtype=torch.float32, device="cuda")
        self.lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
        self.slot = torch.empty(B, dtype=torch.int32, device="cuda")
        self.o_rk, self.o_rv = to_np(c.ring_k).copy(), to_np(c.ring_v).copy()
        self.o_wp, self.o_fill = to_np(c.wp).copy(), to_np(c.fill).copy()
        self.plen = to_np(c.prefix_len).copy()

    def routed(self, s, q_idx):
        c = self.c
        self.rswa.srswa_decode_routed(c.q[s], q_idx, self.kbar, c.pk, c.pv, c.prefix_len, self.ring_k, self.ring_v,
                                      self.wp, self.fill, self.blk, self.logp, self.out, self.ws, lse=self.lse,
                                      tau=self.tau, scale=c.scale)

    def step(self, s, q_idx):
        c = self.c
        self.rswa.srswa_step(c.q[s], c.k_new[s], c.v_new[s], q_idx, self.kbar, c.pk, c.pv, c.prefix_len, self.ring_k,
                             self.ring_v, self.wp, self.fill, self.blk, self.logp, self.out, self.ws, lse=self.lse,
                             tau=self.tau, slot_out=self.slot, scale=c.scale)
        return oracle.append(self.o_rk, self.o_rv, to_np(c.k_new[s]), to_np(c.v_new[s]), self.o_wp, self.o_fill)

    def oracle_decode(self, s, ro):
        sm = self.sample
        c = self.c
        sel = torch.as_tensor(sm, device="cuda")
        return oracle.srswa_decode(to_np(c.q[s])[sm], to_np(c.pk.index_select(0, sel)), to_np(c.pv.index_select(0, sel)),
                                   self.plen[sm], np.ascontiguousarray(ro["blk_idx"][sm]),
                                   np.ascontiguousarray(ro["blk_logp"][sm]), np.ascontiguousarray(self.o_rk[sm]),
                                   np.ascontiguousarray(self.o_rv[sm]), self.o_wp[sm].copy(), self.o_fill[sm].copy(),
                                   c.scale)

    def check_route_exact(self, ro, what):
        np.testing.assert_array_equal(to_np(self.blk), ro["blk_idx"], err_msg=what)
        np.testing.assert_allclose(np.exp(to_np(self.logp)), np.exp(ro["blk_logp"]), rtol=0, atol=ROUTER_P_ABS,
                                   err_msg=what)
        np.testing.assert_allclose(to_np(self.tau), ro["tau"], rtol=0, atol=ROUTER_P_ABS, err_msg=what)

    def check_attention(self, s, ro, what):
        ref, ref_lse = self.oracle_decode(s, ro)
        sm = self.sample
        assert_attention_close(to_np(self.out)[sm], ref, what)
        assert np.abs(to_np(self.lse)[sm] - ref_lse).max() <= LSE_ABS, what


def _planted(rswa, plen, cap, n_dirs, seed):
    pl = synth.plant_router_keys(plen, cap, n_dirs=n_dirs, seed=seed, device="cuda")
    plen_t = torch.tensor(plen, dtype=torch.int32, device="cuda")
    kbar = torch.empty((len(plen), (cap + 31) // 32, 32), dtype=torch.float32, device="cuda")
    rswa.srswa_index_pool(pl.k_idx, plen_t, kbar)
    o_kbar = oracle.index_pool(to_np(pl.k_idx), np.array(plen, np.int32))
    return pl, kbar, o_kbar


def _assert_margins(ro, plen):
    for b, m in enumerate(plen):
        nb = (m + 31) // 32
        zs = np.sort(ro["z"][b, :nb])[::-1]
        assert np.min(zs[:min(16, nb - 1)] - zs[1:min(17, nb)]) >= 1e-3


@pytest.mark.parametrize("plen,H", [
    ([32 * 40, 32 * 23 + 5, 32 * 16, 32 * 200], 4),   # ragged, partial last blocks, a 16-block history
    ([32 * 1024] * 3, 16),                              # 32K histories (16 slices each)
    ([32 * 3200, 8192], 2),                             # the longest history next to a short one
])
def test_routed_planted_matches_oracle(cuda_lib, plen, H):
    cap = max(plen)
    c = synth.decode_case(len(plen), H, 128, plen, cap, 128, 4, seed=611 + H, device="cuda")
    pl, kbar, o_kbar = _planted(cuda_lib, plen, cap, 4, 612 + H)
    f = Fused(cuda_lib, c, kbar)
    for s in range(4):
        f.routed(s, pl.q_idx[s])
        ro = oracle.route(to_np(pl.q_idx[s]), o_kbar, np.array(plen, np.int32))
        _assert_margins(ro, plen)
        f.check_route_exact(ro, f"planted route {s}")
        np.testing.assert_array_equal(to_np(f.blk), to_np(pl.planted[s]))
        f.check_attention(s, ro, f"routed decode {s}")
    assert cuda_lib.check_status(f.ws) == 0


@pytest.mark.parametrize("seed,nb,spread", [
    (1, 1000, 1.0),    # a few hundred candidates
    (2, 3000, 0.2),    # thousands of candidates
    (3, 64, 3.0),      # fewer candidates than topk: the slices' own top lists join them
    (4, 8192, 0.02),   # every block a candidate, at the router's block limit
])
def test_routed_random_scores(cuda_lib, seed, nb, spread):
    rng = np.random.default_rng(seed)
    B = 3
    kbar_np = rng.normal(0, spread, (B, nb, 32)).astype(np.float32)
    q_np = rng.normal(0, 1, (B, 32)).astype(np.float32)
    plen = [nb * 32, nb * 32 - 31, nb * 16]
    c = synth.decode_case(B, 2, 128, plen, nb * 32, 64, 1, seed=620 + seed, device="cuda")
    f = Fused(cuda_lib, c, torch.from_numpy(kbar_np).cuda())
    f.routed(0, torch.from_numpy(q_np).cuda())
    r = oracle.route(q_np, kbar_np.astype(np.float64), np.array(plen, np.int32))
    np.testing.assert_allclose(to_np(f.tau), r["tau"], rtol=0, atol=ROUTER_P_ABS)
    blk, logp = to_np(f.blk), to_np(f.logp)
    for b in range(B):
        z = r["z"][b]
        nbb = (plen[b] + 31) // 32
        assert len(set(blk[b].tolist())) == 16 and blk[b].min() >= 0 and blk[b].max() < nbb
        np.testing.assert_allclose(np.sort(z[blk[b]])[::-1], np.sort(z[:nbb])[::-1][:16], rtol=0, atol=1e-5)
        assert (np.diff(z[blk[b]]) <= 1e-5).all()
        np.testing.assert_allclose(np.exp(logp[b]), r["probs"][b][blk[b]], rtol=0, atol=ROUTER_P_ABS)
    # the attention over the GPU's own route equals the oracle decode over that route
    ro = {"blk_idx": blk, "blk_logp": logp.astype(np.float64)}
    f.check_attention(0, ro, "routed decode, random scores")
    assert cuda_lib.check_status(f.ws) == 0


def test_routed_ties_short_and_empty_histories(cuda_lib):
    nb_cap = 20
    kbar = np.zeros((3, nb_cap, 32), np.float32)
    kbar[0, :, 0] = [1, 3, 3, 2, 3, 0, 1, 1, 2, 2, 3, 3, 3, 0, 0, 0, 1, 2, 3, 3]
    kbar[1, :3, 0] = [0.5, 0.25, 0.75]
    q = np.zeros((3, 32), np.float32)
    q[:, 0] = 1.0
    plen = [20 * 32, 3 * 32 - 4, 0]
    c = synth.decode_case(3, 2, 128, plen, nb_cap * 32, 16, 1, seed=631, device="cuda", fill0=[16, 5, 16])
    f = Fused(cuda_lib, c, torch.from_numpy(kbar).cuda(), topk=8)
    f.routed(0, torch.from_numpy(q).cuda())
    r = oracle.route(q, kbar.astype(np.float64), np.array(plen, np.int32), topk=8)
    blk = to_np(f.blk)
    np.testing.assert_array_equal(blk, r["blk_idx"])
    np.testing.assert_array_equal(blk[0], [1, 2, 4, 10, 11, 12, 18, 19])
    np.testing.assert_array_equal(blk[1], [2, 0, 1, -1, -1, -1, -1, -1])
    assert (blk[2] == -1).all() and np.isneginf(to_np(f.logp)[2]).all() and np.isnan(to_np(f.tau)[2])
    f.check_attention(0, r, "ties / short / empty")       # the empty history attends to its ring only
    assert cuda_lib.check_status(f.ws) == 0


def _fused_steps(rswa, plen, cap, B, H, steps, sample, seed):
    c = synth.decode_case(B, H, 128, plen, cap, 128, steps, seed=seed, device="cuda")
    pl, kbar, o_kbar = _planted(rswa, plen, cap, steps, seed + 1)
    f = Fused(rswa, c, kbar, sample=sample)
    for s in range(steps):
        o_slot = f.step(s, pl.q_idx[s])
        ro = oracle.route(to_np(pl.q_idx[s]), o_kbar, np.array(plen, np.int32))
        np.testing.assert_array_equal(to_np(f.slot), o_slot, err_msg=f"slot_out step {s}")
        np.testing.assert_array_equal(to_np(f.wp), f.o_wp, err_msg=f"wp step {s}")
        np.testing.assert_array_equal(to_np(f.fill), f.o_fill, err_msg=f"fill step {s}")
        f.check_route_exact(ro, f"step {s}")
        f.check_attention(s, ro, f"fused step {s}")
    sel = torch.as_tensor(f.sample, device="cuda")
    np.testing.assert_array_equal(to_np(f.ring_k.index_select(0, sel)), f.o_rk[f.sample])
    np.testing.assert_array_equal(to_np(f.ring_v.index_select(0, sel)), f.o_rv[f.sample])
    assert rswa.check_status(f.ws) == 0


def test_step_small_rings_wrap(cuda_lib):
    # empty and partial rings that fill and wrap over 40 steps, ragged prefixes
    plen = [32 * 20 + 7, 32 * 17, 32 * 64]
    cap = 32 * 64
    c = synth.decode_case(3, 4, 128, plen, cap, 24, 40, seed=641, device="cuda", wp0=[0, 5, 23], fill0=[0, 9, 24])
    pl, kbar, o_kbar = _planted(cuda_lib, plen, cap, 32, 642)
    f = Fused(cuda_lib, c, kbar)
    for s in range(40):
        o_slot = f.step(s, pl.q_idx[s % 32])
        ro = oracle.route(to_np(pl.q_idx[s % 32]), o_kbar, np.array(plen, np.int32))
        np.testing.assert_array_equal(to_np(f.slot), o_slot)
        f.check_route_exact(ro, f"step {s}")
        f.check_attention(s, ro, f"step {s}")
    np.testing.assert_array_equal(to_np(f.ring_k), f.o_rk)
    np.testing.assert_array_equal(to_np(f.ring_v), f.o_rv)
    np.testing.assert_array_equal(to_np(f.wp), f.o_wp)
    np.testing.assert_array_equal(to_np(f.fill), f.o_fill)
    assert cuda_lib.check_status(f.ws) == 0


def test_step_32k_history_sampled(cuda_lib):
    # 64 sequences of 32768 tokens: the benchmark's SR-SWA shape; oracle decode on 8 sequences
    _fused_steps(cuda_lib, [32768] * 64, 32768, 64, 16, 3, np.arange(0, 64, 8), seed=4101)


def test_step_ragged_long_horizon_sampled(cuda_lib):
    # 16 sequences, 8192..102400 tokens (log-uniform page counts x 256)
    pages = synth.log_uniform_pages(16, 32, 400, seed=5005)
    plen = [256 * p for p in pages]
    sample = np.array(sorted({int(np.argmax(plen)), int(np.argmin(plen)), 5, 11}))
    _fused_steps(cuda_lib, plen, 102400, 16, 16, 3, sample, seed=5101)
