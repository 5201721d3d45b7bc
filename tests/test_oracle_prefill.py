"""Pins of the oracle's chunked R-SWA prefill.

- brute force over the explicit R-SWA mask ([R-SWA tutorial] §3.3.1):
  every reference row visible, output j visible to query i iff i - n < j <= i;
- n >= T with an empty ring is causal attention over [prefix; outputs] with the
  prefix fully visible (torch scaled_dot_product_attention with a causal mask);
- row i equals a decode step after appending outputs 0..i;
- a chunk split in two (the second reading the first through the ring) equals
  one chunk.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.bruteforce import masked_attention, rswa_visible, u16_to_f64


def _np(d):
    return {k: (synth.to_u16(v) if isinstance(v, torch.Tensor) and v.dtype == torch.bfloat16 else
                (v.cpu().numpy() if isinstance(v, torch.Tensor) else v)) for k, v in d.items()}


@pytest.mark.parametrize("plen,n,T", [([7, 3], 4, 12), ([0, 5], 3, 9), ([12, 12], 16, 10)])
def test_prefill_bruteforce(plen, n, T):
    B, H, D = 2, 2, 128
    a = _np(synth.prefill_case(B, H, D, plen, 12, T, seed=21))
    rows = np.arange(T, dtype=np.int32)
    out, lse = oracle.rswa_prefill(a["q"], a["k_out"], a["v_out"], a["pk"], a["pv"], a["prefix_len"], a["scale"],
                                   rows, n)
    for b in range(B):
        m = plen[b]
        for h in range(H):
            K = torch.cat([u16_to_f64(a["pk"][b, h, :m]), u16_to_f64(a["k_out"][b, h])])
            V = torch.cat([u16_to_f64(a["pv"][b, h, :m]), u16_to_f64(a["v_out"][b, h])])
            ref, ref_lse = masked_attention(u16_to_f64(a["q"][b, h]), K, V, rswa_visible(m, n, list(range(T)), T),
                                            a["scale"])
            np.testing.assert_allclose(out[b, h], ref.numpy(), rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], ref_lse.numpy(), rtol=0, atol=1e-12)


def test_prefill_n_ge_T_is_causal_attention_with_visible_prefix():
    B, H, D, T, m, n = 1, 3, 128, 24, 10, 128
    a = _np(synth.prefill_case(B, H, D, m, m, T, seed=22))
    rows = np.arange(T, dtype=np.int32)
    out, _ = oracle.rswa_prefill(a["q"], a["k_out"], a["v_out"], a["pk"], a["pv"], a["prefix_len"], a["scale"],
                                 rows, n)
    mask = torch.ones((T, m + T), dtype=torch.bool)
    mask[:, m:] = torch.tril(torch.ones((T, T), dtype=torch.bool))
    for h in range(H):
        K = torch.cat([u16_to_f64(a["pk"][0, h]), u16_to_f64(a["k_out"][0, h])])
        V = torch.cat([u16_to_f64(a["pv"][0, h]), u16_to_f64(a["v_out"][0, h])])
        ref = torch.nn.functional.scaled_dot_product_attention(u16_to_f64(a["q"][0, h])[None], K[None], V[None],
                                                               attn_mask=mask, scale=a["scale"])
        np.testing.assert_allclose(out[0, h], ref[0].numpy(), rtol=0, atol=1e-12)


def test_prefill_row_equals_decode_step():
    B, H, D, T, m, n = 2, 2, 128, 14, 9, 5
    a = _np(synth.prefill_case(B, H, D, m, m, T, seed=23))
    rows = np.arange(T, dtype=np.int32)
    out, lse = oracle.rswa_prefill(a["q"], a["k_out"], a["v_out"], a["pk"], a["pv"], a["prefix_len"], a["scale"],
                                   rows, n)
    ring_k = np.zeros((B, H, n, D), np.uint16)
    ring_v = np.zeros((B, H, n, D), np.uint16)
    wp = np.zeros(B, np.int32)
    fill = np.zeros(B, np.int32)
    for i in range(T):
        oracle.append(ring_k, ring_v, a["k_out"][:, :, i], a["v_out"][:, :, i], wp, fill)
        o, l = oracle.rswa_decode(a["q"][:, :, i], a["pk"], a["pv"], a["prefix_len"], ring_k, ring_v, wp, fill,
                                  a["scale"])
        np.testing.assert_allclose(out[:, :, i], o, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], l, rtol=0, atol=1e-13)


@pytest.mark.parametrize("T1", [3, 5, 8])
def test_prefill_two_chunks_equal_one(T1):
    B, H, D, T, m, n = 2, 2, 128, 13, 7, 5
    a = _np(synth.prefill_case(B, H, D, [7, 4], m, T, seed=24))
    rows = np.arange(T, dtype=np.int32)
    full, full_lse = oracle.rswa_prefill(a["q"], a["k_out"], a["v_out"], a["pk"], a["pv"], a["prefix_len"],
                                         a["scale"], rows, n)
    # chunk 1's outputs go through the ring (append in order), chunk 2 reads them from there
    ring_k = np.zeros((B, H, n, D), np.uint16)
    ring_v = np.zeros((B, H, n, D), np.uint16)
    wp = np.array([2, 0], np.int32)   # an empty ring may start at any slot
    fill = np.zeros(B, np.int32)
    for i in range(T1):
        oracle.append(ring_k, ring_v, a["k_out"][:, :, i], a["v_out"][:, :, i], wp, fill)
    sl = slice(T1, T)
    q2, k2, v2 = (np.ascontiguousarray(a[x][:, :, sl]) for x in ("q", "k_out", "v_out"))
    part, part_lse = oracle.rswa_prefill(q2, k2, v2, a["pk"], a["pv"], a["prefix_len"], a["scale"],
                                         np.arange(T - T1, dtype=np.int32), n, ring_k, ring_v, wp, fill)
    np.testing.assert_allclose(part, full[:, :, sl], rtol=0, atol=1e-13)
    np.testing.assert_allclose(part_lse, full_lse[:, :, sl], rtol=0, atol=1e-13)
