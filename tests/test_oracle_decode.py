"""Pins of the oracle's ring append and R-SWA decode against what the pages fix.

- slot/fill closed form: the write pointer advances cyclically, so the s-th
  append writes slot (wp0 + s) mod n, and the cache holds L_m + min(n, T)
  tokens ([R-SWA summary] §二.2).
- ring contents: a deque(maxlen=n) of the appended tokens, oldest first
  ([R-SWA tutorial] §3.3.2).
- decode: brute force over an explicit R-SWA mask on the flat token timeline
  ([R-SWA tutorial] §3.3.1), the n >= T reduction to full causal attention
  (torch scaled_dot_product_attention), m = 0 with one token, constant V.
"""
from collections import deque

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.bruteforce import masked_attention, rswa_visible, u16_to_f64


def _np(c):
    return {k: (synth.to_u16(v) if v.dtype == torch.bfloat16 else v.cpu().numpy())
            for k, v in c.__dict__.items() if isinstance(v, torch.Tensor)}


@pytest.mark.parametrize("n,wp0,fill0", [(4, 0, 0), (4, 3, 0), (7, 5, 7), (128, 37, 128), (5, 2, 3)])
def test_append_closed_form_and_deque(n, wp0, fill0):
    B, H, D, T = 2, 3, 8, 3 * n + 2
    c = synth.decode_case(B, H, D, 4, 4, n, T, seed=11, wp0=wp0, fill0=fill0)
    a = _np(c)
    ring_k, ring_v = a["ring_k"].copy(), a["ring_v"].copy()
    wp, fill = a["wp"].copy(), a["fill"].copy()
    # the deque starts with the valid initial slots, oldest first
    dq = [deque(maxlen=n) for _ in range(B * H)]
    for b in range(B):
        for h in range(H):
            for i in range(fill0):
                dq[b * H + h].append(a["ring_k"][b, h, (wp0 - fill0 + i) % n].copy())
    for s in range(T):
        slot = oracle.append(ring_k, ring_v, a["k_new"][s], a["v_new"][s], wp, fill)
        assert (slot == (wp0 + s) % n).all()
        assert (wp == (wp0 + s + 1) % n).all()
        assert (fill == min(fill0 + s + 1, n)).all()
        for b in range(B):
            for h in range(H):
                dq[b * H + h].append(a["k_new"][s, b, h].copy())
                got = [ring_k[b, h, (wp[b] - fill[b] + i) % n] for i in range(fill[b])]
                want = list(dq[b * H + h])
                assert len(got) == len(want)
                for g_row, w_row in zip(got, want):
                    assert (g_row == w_row).all()


def test_cache_tokens_closed_form():
    # C_R-SWA(T) = L_m + min(n, T) <= L_m + n, C_MHA(T) = L_m + T
    per_tok = 2 * 16 * 128 * 2
    for T in (0, 1, 64, 127, 128, 129, 5000):
        assert oracle.kv_cache_bytes(288, T, 16, 128, 1, 2, 128) == (288 + min(128, T)) * per_tok
        assert oracle.kv_cache_bytes(288, T, 16, 128, 1, 2, None) == (288 + T) * per_tok
        assert oracle.kv_cache_bytes(288, T, 16, 128, 1, 2, 128) <= (288 + 128) * per_tok


def _run_steps(c, a, steps):
    """Append + decode with the oracle for `steps` steps; returns per-step outputs."""
    ring_k, ring_v = a["ring_k"].copy(), a["ring_v"].copy()
    wp, fill = a["wp"].copy(), a["fill"].copy()
    outs = []
    for s in range(steps):
        oracle.append(ring_k, ring_v, a["k_new"][s], a["v_new"][s], wp, fill)
        outs.append(oracle.rswa_decode(a["q"][s], a["pk"], a["pv"], a["prefix_len"], ring_k, ring_v, wp, fill,
                                       c.scale))
    return outs


@pytest.mark.parametrize("plen,n,wp0", [([5, 3], 4, 0), ([5, 0], 4, 2), ([9, 7], 6, 1)])
def test_decode_bruteforce_mask_from_empty_ring(plen, n, wp0):
    B, H, D, T = 2, 2, 128, 11
    c = synth.decode_case(B, H, D, plen, 9, n, T, seed=5, wp0=wp0, fill0=0)
    a = _np(c)
    outs = _run_steps(c, a, T)
    for b in range(B):
        m = plen[b]
        for h in range(H):
            k_tl = torch.cat([u16_to_f64(a["pk"][b, h, :m]), u16_to_f64(a["k_new"][:, b, h])])
            v_tl = torch.cat([u16_to_f64(a["pv"][b, h, :m]), u16_to_f64(a["v_new"][:, b, h])])
            qs = u16_to_f64(a["q"][:, b, h])
            vis = rswa_visible(m, n, list(range(T)), T)
            ref, ref_lse = masked_attention(qs, k_tl, v_tl, vis, c.scale)
            for t in range(T):
                got, got_lse = outs[t]
                np.testing.assert_allclose(got[b, h], ref[t].numpy(), rtol=0, atol=1e-12)
                assert abs(got_lse[b, h] - ref_lse[t].item()) < 1e-12


def test_decode_bruteforce_full_ring_with_history():
    # The ring starts full: its slots hold outputs -n..-1 (oldest at wp0).
    B, H, D, n, T, m = 1, 2, 128, 5, 13, 6
    c = synth.decode_case(B, H, D, m, m, n, T, seed=8, wp0=3, fill0=n)
    a = _np(c)
    outs = _run_steps(c, a, T)
    for h in range(H):
        hist_k = [a["ring_k"][0, h, (3 - n + i) % n] for i in range(n)]
        hist_v = [a["ring_v"][0, h, (3 - n + i) % n] for i in range(n)]
        k_tl = torch.cat([u16_to_f64(a["pk"][0, h]), u16_to_f64(np.stack(hist_k)), u16_to_f64(a["k_new"][:, 0, h])])
        v_tl = torch.cat([u16_to_f64(a["pv"][0, h]), u16_to_f64(np.stack(hist_v)), u16_to_f64(a["v_new"][:, 0, h])])
        vis = rswa_visible(m, n, list(range(T)), n + T, first_out=-n)
        ref, _ = masked_attention(u16_to_f64(a["q"][:, 0, h]), k_tl, v_tl, vis, c.scale)
        for t in range(T):
            np.testing.assert_allclose(outs[t][0][0, h], ref[t].numpy(), rtol=0, atol=1e-12)


def test_decode_n_ge_T_is_full_causal_attention():
    # With n >= T nothing is evicted: step t attends to the prefix and every output 0..t.
    B, H, D, n, T, m = 2, 2, 128, 128, 40, 17
    c = synth.decode_case(B, H, D, m, m, n, T, seed=3, wp0=0, fill0=0)
    a = _np(c)
    outs = _run_steps(c, a, T)
    for b in range(B):
        for h in range(H):
            K = torch.cat([u16_to_f64(a["pk"][b, h]), u16_to_f64(a["k_new"][:, b, h])])
            V = torch.cat([u16_to_f64(a["pv"][b, h]), u16_to_f64(a["v_new"][:, b, h])])
            for t in range(T):
                q = u16_to_f64(a["q"][t, b, h])[None, None, None, :]
                ref = torch.nn.functional.scaled_dot_product_attention(
                    q, K[None, None, :m + t + 1], V[None, None, :m + t + 1], scale=c.scale)
                np.testing.assert_allclose(outs[t][0][b, h], ref[0, 0, 0].numpy(), rtol=0, atol=1e-12)


def test_decode_single_key_returns_v_self():
    B, H, D, n = 3, 2, 128, 8
    c = synth.decode_case(B, H, D, 0, 1, n, 1, seed=9, wp0=[0, 4, 7], fill0=0)
    a = _np(c)
    (out, lse), = _run_steps(c, a, 1)
    v_self = u16_to_f64(a["v_new"][0]).numpy()
    assert (out == v_self).all()
    qk = (u16_to_f64(a["q"][0]) * u16_to_f64(a["k_new"][0])).sum(-1).numpy()
    np.testing.assert_allclose(lse, c.scale * qk, rtol=0, atol=1e-12)


def test_decode_constant_v():
    B, H, D, n, m = 2, 2, 128, 8, 20
    c = synth.decode_case(B, H, D, m, m, n, 4, seed=4, wp0=1, fill0=n)
    const = torch.tensor(0.71875, dtype=torch.bfloat16)
    c.pv.fill_(const)
    c.ring_v.fill_(const)
    c.v_new.fill_(const)
    a = _np(c)
    for out, _ in _run_steps(c, a, 4):
        np.testing.assert_allclose(out, 0.71875, rtol=1e-15, atol=0)
