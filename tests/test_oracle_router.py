"""Pins of the oracle's SR-SWA router (index pooling, 1.5-entmax, top-k, log
bias) and gathered-block decode.

- entmax: the sort-based threshold equals a bisection solve of
  sum max(x - tau, 0)^2 = 1; p >= 0 and sums to 1; two inputs follow the
  closed form p1 = ((d + sqrt(2 - d^2)) / 2)^2 for a gap d < 1 and (1, 0) for
  d >= 1; equal inputs give the uniform distribution; adding a constant to
  every input changes nothing.
- pooling: constant blocks, antithetic pairs and a partial last block whose
  invalid tail holds NaN give exact means.
- top-k: the planted top-16 of every query direction comes back in order; equal
  scores rank the smaller block first; fewer than k blocks pad with -1.
- SR-SWA decode: every block selected with zero bias equals R-SWA decode; a
  uniform bias over the selected blocks with an empty ring is a no-op; a dense
  biased softmax on tiny inputs.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.bruteforce import entmax15_bisect, masked_attention, u16_to_f64


@pytest.mark.parametrize("seed,K,spread", [(0, 1, 1.0), (1, 2, 0.3), (2, 7, 1.0), (3, 100, 0.2), (4, 1000, 3.0),
                                           (5, 3000, 0.05), (6, 64, 10.0)])
def test_entmax_sort_equals_bisection(seed, K, spread):
    x = np.random.default_rng(seed).normal(0, spread, K)
    p, tau = oracle.entmax15(x)
    pb, taub = entmax15_bisect(x)
    assert abs(tau - taub) < 1e-12
    np.testing.assert_allclose(p, pb, rtol=0, atol=1e-12)
    assert (p >= 0).all()
    assert abs(p.sum() - 1.0) < 1e-12


@pytest.mark.parametrize("d", [0.0, 0.1, 0.5, 0.9, 0.999])
def test_entmax_two_element_closed_form(d):
    p, _ = oracle.entmax15(np.array([0.3 + d, 0.3]))
    r = math.sqrt(2 - d * d)
    assert abs(p[0] - ((d + r) / 2) ** 2) < 1e-14
    assert abs(p[1] - ((-d + r) / 2) ** 2) < 1e-14


@pytest.mark.parametrize("d", [1.0, 1.5, 7.0])
def test_entmax_two_element_gap_ge_one_is_onehot(d):
    p, _ = oracle.entmax15(np.array([-0.2, -0.2 + d]))
    assert p[1] == 1.0 and p[0] == 0.0


@pytest.mark.parametrize("K", [1, 3, 16, 1024])
def test_entmax_uniform(K):
    p, tau = oracle.entmax15(np.full(K, 0.37))
    np.testing.assert_allclose(p, 1.0 / K, rtol=1e-10)
    assert abs(tau - (0.37 - math.sqrt(1.0 / K))) < 1e-11


@pytest.mark.parametrize("shift,tol", [(7.75, 1e-11), (123.25, 1e-8)])
def test_entmax_shift_invariance(shift, tol):
    # the sums of squares grow with the shift, so fp64 cancellation grows too
    x = np.random.default_rng(7).normal(0, 0.7, 200)
    p0, t0 = oracle.entmax15(x)
    p1, t1 = oracle.entmax15(x + shift)
    np.testing.assert_allclose(p0, p1, rtol=0, atol=tol)
    assert abs((t1 - t0) - shift) < tol


def _bf16_bits(x):
    return synth.to_u16(torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16))


def test_index_pool_exact_means():
    B, cap, DI, blk = 2, 100, 32, 32
    rng = np.random.default_rng(3)
    keys = np.zeros((B, cap, DI), np.float32)
    plen = np.array([100, 70], np.int32)
    # block 0: constant rows; block 1: antithetic pairs around a centre; blocks 2+: random
    keys[:, 0:32] = 0.5
    centre = np.round(rng.normal(0, 1, (B, DI)) * 8) / 8
    e = np.round(rng.normal(0, 1, (B, 16, DI)) * 8) / 8
    keys[:, 32:64:2] = centre[:, None] + e
    keys[:, 33:64:2] = centre[:, None] - e
    keys[:, 64:] = np.round(rng.normal(0, 1, (B, cap - 64, DI)) * 16) / 16
    bits = _bf16_bits(keys)
    bits[1, 70:] = synth.BF16_NAN_BITS          # sequence 1 ends at 70: a 6-token partial block
    kbar = oracle.index_pool(bits, plen, blk)
    assert kbar.shape == (B, 4, DI)
    assert (kbar[:, 0] == 0.5).all()
    np.testing.assert_array_equal(kbar[:, 1], centre.astype(np.float64))
    vals = u16_to_f64(bits).numpy()
    np.testing.assert_allclose(kbar[0, 3], vals[0, 96:100].sum(0) / 4, rtol=1e-15)
    np.testing.assert_allclose(kbar[1, 2], vals[1, 64:70].sum(0) / 6, rtol=1e-15)
    assert (kbar[1, 3] == 0).all() and np.isfinite(kbar).all()


def test_route_planted_top16_and_entmax_support():
    plen = [32 * 40, 32 * 23 + 5, 32 * 16, 32 * 200]
    cap = max(plen)
    pl = synth.plant_router_keys(plen, cap, n_dirs=5, seed=31)
    k_idx = synth.to_u16(pl.k_idx)
    plen_np = np.array(plen, np.int32)
    kbar = oracle.index_pool(k_idx, plen_np)
    for s in range(pl.n_dirs):
        r = oracle.route(pl.q_idx[s].numpy(), kbar, plen_np, topk=16)
        np.testing.assert_array_equal(r["blk_idx"], pl.planted[s].numpy())
        for b, m in enumerate(plen):
            nb = (m + 31) // 32
            z = r["z"][b, :nb]
            zs = np.sort(z)[::-1]
            gaps = zs[:min(16, nb - 1)] - zs[1:min(17, nb)]
            assert np.min(gaps) >= 1e-3                           # margins of the planted top-16
            p = r["probs"][b, :nb]
            assert set(np.nonzero(p)[0]) == set(pl.planted[s, b].tolist())   # support = planted blocks
            assert abs(p.sum() - 1) < 1e-12
            np.testing.assert_allclose(r["blk_logp"][b], np.log(p[r["blk_idx"][b]]), rtol=0, atol=1e-12)
            _, tb = entmax15_bisect(z / 2)
            assert abs(r["tau"][b] - tb) < 1e-12


def test_route_ties_and_short_history():
    DI = 32
    kbar = np.zeros((2, 20, DI))
    kbar[0, :, 0] = np.array([1, 3, 3, 2, 3, 0, 1, 1, 2, 2, 3, 3, 3, 0, 0, 0, 1, 2, 3, 3], np.float64)
    kbar[1, :3, 0] = [0.5, 0.25, 0.75]
    q = np.zeros((2, DI), np.float32)
    q[:, 0] = 1.0
    plen = np.array([20 * 32, 3 * 32 - 4], np.int32)
    r = oracle.route(q, kbar, plen, topk=8)
    np.testing.assert_array_equal(r["blk_idx"][0], [1, 2, 4, 10, 11, 12, 18, 19])
    np.testing.assert_array_equal(r["blk_idx"][1], [2, 0, 1, -1, -1, -1, -1, -1])
    assert np.isneginf(r["blk_logp"][1, 3:]).all()


def _decode_np(c):
    return {k: (synth.to_u16(v) if v.dtype == torch.bfloat16 else v.cpu().numpy())
            for k, v in c.__dict__.items() if isinstance(v, torch.Tensor)}


def test_srswa_all_blocks_zero_bias_equals_rswa():
    B, H, D, n = 2, 2, 128, 8
    plen = [32 * 5, 32 * 3 + 7]
    c = synth.decode_case(B, H, D, plen, 32 * 5, n, 1, seed=41, wp0=[1, 6], fill0=[8, 5])
    a = _decode_np(c)
    blk_idx = np.array([[3, 0, 4, 1, 2], [1, 3, 0, 2, -1]], np.int32)
    logp = np.zeros((B, 5))
    logp[1, 4] = -np.inf
    o1, l1 = oracle.srswa_decode(a["q"][0], a["pk"], a["pv"], a["prefix_len"], blk_idx, logp, a["ring_k"],
                                 a["ring_v"], a["wp"], a["fill"], c.scale)
    o2, l2 = oracle.rswa_decode(a["q"][0], a["pk"], a["pv"], a["prefix_len"], a["ring_k"], a["ring_v"], a["wp"],
                                a["fill"], c.scale)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l2, rtol=0, atol=1e-12)


def test_srswa_uniform_bias_without_ring_is_noop():
    B, H, D, n = 1, 3, 128, 4
    c = synth.decode_case(B, H, D, 32 * 20, 32 * 20, n, 1, seed=42, wp0=0, fill0=0)
    a = _decode_np(c)
    sel = np.array([[19, 4, 7, 0, 11, 2, 9, 13, 5, 6, 1, 17, 8, 3, 15, 10]], np.int32)
    o0, l0 = oracle.srswa_decode(a["q"][0], a["pk"], a["pv"], a["prefix_len"], sel, np.zeros((1, 16)), a["ring_k"],
                                 a["ring_v"], a["wp"], a["fill"], c.scale)
    o1, l1 = oracle.srswa_decode(a["q"][0], a["pk"], a["pv"], a["prefix_len"], sel, np.full((1, 16), math.log(1 / 16)),
                                 a["ring_k"], a["ring_v"], a["wp"], a["fill"], c.scale)
    np.testing.assert_allclose(o0, o1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1, l0 + math.log(1 / 16), rtol=0, atol=1e-12)


def test_srswa_bruteforce_dense_biased_softmax():
    B, H, D, n = 2, 2, 128, 6
    plen = [32 * 6 + 9, 32 * 4]
    c = synth.decode_case(B, H, D, plen, 32 * 7, n, 1, seed=43, wp0=[2, 5], fill0=[6, 3])
    a = _decode_np(c)
    sel = np.array([[6, 2, 0], [3, 1, -1]], np.int32)
    logp = np.array([[-0.5, -1.25, -3.0], [-0.1, -np.inf, -np.inf]])
    out, lse = oracle.srswa_decode(a["q"][0], a["pk"], a["pv"], a["prefix_len"], sel, logp, a["ring_k"], a["ring_v"],
                                   a["wp"], a["fill"], c.scale)
    for b in range(B):
        m = plen[b]
        for h in range(H):
            # dense: every prefix row and every ring slot, with bias -inf where not visible
            K = torch.cat([u16_to_f64(a["pk"][b, h, :m]), u16_to_f64(a["ring_k"][b, h])])
            V = torch.cat([u16_to_f64(a["pv"][b, h, :m]), u16_to_f64(a["ring_v"][b, h])])
            bias = torch.full((m + n,), float("-inf"), dtype=torch.float64)
            for c_blk, lp in zip(sel[b], logp[b]):
                if c_blk >= 0:
                    bias[32 * c_blk:min(32 * c_blk + 32, m)] = lp
            fill, wp = int(a["fill"][b]), int(a["wp"][b])
            for i in range(fill):
                bias[m + (wp - fill + i) % n] = 0.0
            vis = torch.isfinite(bias)[None, :]
            ref, ref_lse = masked_attention(u16_to_f64(a["q"][0, b, h])[None], K, V, vis, c.scale, bias)
            np.testing.assert_allclose(out[b, h], ref[0].numpy(), rtol=0, atol=1e-12)
            assert abs(lse[b, h] - ref_lse[0].item()) < 1e-12
