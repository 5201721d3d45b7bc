"""Pins of the oracle's FP8 (E4M3) ring: the append that quantises each written row,
and the R-SWA / SR-SWA decodes over an FP8 prefix and an FP8 ring.

- append: slots, wp and fill follow oracle.append's (separately pinned) recurrence on the
  same inputs, through wrap-around and a filling ring; every written row equals the prefix
  quantiser (separately pinned against the E4M3 format and an exhaustive encoder search)
  applied to that row as a one-row block; rows not written keep their bytes.
- decodes: on data on the E4M3 grid with a 448 in every prefix block and every ring row,
  each block and row then multiplied by its own power of two (so every scale is that
  power of two and every element is exactly its code value times its scale), the FP8
  decodes equal the bf16 decodes of the same values exactly, with a full wrapped ring and
  with a partly filled one; on N(0, 1) data they track the bf16 decodes to quantisation
  error.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.test_oracle_fp8 import GRID_POW2, _grid_prefix, _table


def _bf16(shape, seed, scale=1.0):
    return oracle.bf16_round(np.random.default_rng(seed).standard_normal(shape) * scale)


def test_append_fp8_recurrence_and_rows():
    B, H, n, D = 3, 2, 5, 128
    rk8, rv8, rks, rvs = oracle.fp8_ring(B, H, n, D)
    ring_k = np.zeros((B, H, n, D), np.uint16)
    ring_v = np.zeros((B, H, n, D), np.uint16)
    wp = np.array([0, 3, 4], np.int32)
    fill = np.array([0, 5, 2], np.int32)
    wp_b, fill_b = wp.copy(), fill.copy()
    for s in range(13):                                        # wraps the 5-slot ring twice
        k = _bf16((B, H, D), 100 + s, scale=np.exp(s % 5 - 2))
        v = _bf16((B, H, D), 200 + s)
        before_k, before_v = rk8.copy(), rv8.copy()
        slot = oracle.append_fp8(rk8, rv8, rks, rvs, k, v, wp, fill)
        slot_b = oracle.append(ring_k, ring_v, k, v, wp_b, fill_b)
        np.testing.assert_array_equal(slot, slot_b)
        np.testing.assert_array_equal(wp, wp_b)
        np.testing.assert_array_equal(fill, fill_b)
        for b in range(B):
            # the written row is the prefix quantiser's one-row block
            want8, wants = oracle.quantize_prefix(k[b][None, :, None, :].copy(), np.array([1], np.int32), blk=1)
            np.testing.assert_array_equal(rk8[b, :, slot[b]], want8[0, :, 0])
            np.testing.assert_array_equal(rks[b, :, slot[b]], wants[0, :, 0])
            want8, wants = oracle.quantize_prefix(v[b][None, :, None, :].copy(), np.array([1], np.int32), blk=1)
            np.testing.assert_array_equal(rv8[b, :, slot[b]], want8[0, :, 0])
            np.testing.assert_array_equal(rvs[b, :, slot[b]], wants[0, :, 0])
            others = np.arange(n) != slot[b]
            np.testing.assert_array_equal(rk8[b][:, others], before_k[b][:, others])
            np.testing.assert_array_equal(rv8[b][:, others], before_v[b][:, others])


def _grid_rows(shape, seed, pow2=None):
    """bf16 rows of E4M3 values with a 448 in every row, each row times 2^e (e from pow2, an
    integer array of the rows' shape): the row's scale is then exactly 2^e and every element
    is its code value times that scale, exactly."""
    rng = np.random.default_rng(seed)
    t = _table()
    codes = rng.integers(0, 0x7f, shape).astype(np.uint8) | (rng.integers(0, 2, shape) << 7).astype(np.uint8)
    codes[..., 0] = 0x7e
    vals = t[codes] * (np.exp2(pow2)[..., None] if pow2 is not None else 1.0)
    return synth.to_u16(torch.from_numpy(vals.astype(np.float32)).bfloat16())


def _fp8_inputs(B, H, D, n, cap, plen, seed, grid, appends=None):
    """A prefix (quantised by blocks), a ring filled by `appends` calls of append_fp8 (default
    n + 3: full and wrapped) and its bf16 twin, one query. grid: E4M3-grid data with
    power-of-two block and row scales, so that the FP8 data equal the bf16 data exactly."""
    c = synth.decode_case(B, H, D, plen, cap, n, 1, seed=seed, wp0=2, fill0=0)
    if grid:
        pk = synth.to_u16(_grid_prefix(B, H, cap, D, seed + 1)[0])
        pv = synth.to_u16(_grid_prefix(B, H, cap, D, seed + 2)[0])
    else:
        pk, pv = synth.to_u16(c.pk), synth.to_u16(c.pv)
    p = np.array(plen, np.int32)
    k8, ks = oracle.quantize_prefix(pk, p)
    v8, vs = oracle.quantize_prefix(pv, p)
    rk8, rv8, rks, rvs = oracle.fp8_ring(B, H, n, D)
    ring_k = np.zeros((B, H, n, D), np.uint16)
    ring_v = np.zeros((B, H, n, D), np.uint16)
    wp, fill = c.wp.numpy().copy(), c.fill.numpy().copy()
    wp8, fill8 = wp.copy(), fill.copy()
    rng = np.random.default_rng(seed + 5)
    for s in range(n + 3 if appends is None else appends):
        if grid:
            k = _grid_rows((B, H, D), 300 + s, rng.integers(GRID_POW2[0], GRID_POW2[1] + 1, (B, H)))
            v = _grid_rows((B, H, D), 400 + s, rng.integers(GRID_POW2[0], GRID_POW2[1] + 1, (B, H)))
        else:
            k, v = _bf16((B, H, D), 300 + s), _bf16((B, H, D), 400 + s)
        oracle.append_fp8(rk8, rv8, rks, rvs, k, v, wp8, fill8)
        oracle.append(ring_k, ring_v, k, v, wp, fill)
    if grid:   # written scales are powers of two that differ between rows, K and V
        assert np.all(np.log2(rks) % 1 == 0) and np.all(np.log2(rvs) % 1 == 0)
        assert len(np.unique(rks)) > 3 and not np.array_equal(rks, rvs)
    q = synth.to_u16(c.q[0])
    return dict(q=q, pk=pk, pv=pv, p=p, k8=k8, v8=v8, ks=ks, vs=vs, ring=(ring_k, ring_v, wp, fill),
                ring8=(rk8, rv8, rks, rvs, wp8, fill8), scale=c.scale)


@pytest.mark.parametrize("appends", [None, 5])           # a full, wrapped ring; a partly filled one
def test_rswa_decode_fp8kv_equals_bf16_on_grid_data(appends):
    d = _fp8_inputs(2, 2, 128, 8, 96, [96, 70], seed=31, grid=True, appends=appends)
    ref, ref_lse = oracle.rswa_decode(d["q"], d["pk"], d["pv"], d["p"], *d["ring"], d["scale"])
    got, got_lse = oracle.rswa_decode_fp8kv(d["q"], d["k8"], d["v8"], d["ks"], d["vs"], d["p"], *d["ring8"],
                                            d["scale"])
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(got_lse, ref_lse)


@pytest.mark.parametrize("appends", [None, 3])
def test_srswa_decode_fp8kv_equals_bf16_on_grid_data(appends):
    d = _fp8_inputs(2, 2, 128, 8, 160, [160, 100], seed=32, grid=True, appends=appends)
    blk = np.array([[4, 0, 2, -1], [3, 1, 0, 2]], np.int32)
    logp = np.log(np.array([[0.5, 0.3, 0.2, 1.0], [0.4, 0.3, 0.2, 0.1]]))
    ref, ref_lse = oracle.srswa_decode(d["q"], d["pk"], d["pv"], d["p"], blk, logp, *d["ring"], d["scale"])
    got, got_lse = oracle.srswa_decode_fp8kv(d["q"], d["k8"], d["v8"], d["ks"], d["vs"], d["p"], blk, logp,
                                             *d["ring8"], d["scale"])
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(got_lse, ref_lse)


def test_fp8kv_decode_tracks_bf16_decode_on_gaussian_data():
    d = _fp8_inputs(2, 2, 128, 16, 256, [256, 190], seed=33, grid=False)
    ref, _ = oracle.rswa_decode(d["q"], d["pk"], d["pv"], d["p"], *d["ring"], d["scale"])
    got, _ = oracle.rswa_decode_fp8kv(d["q"], d["k8"], d["v8"], d["ks"], d["vs"], d["p"], *d["ring8"], d["scale"])
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert 0 < rel < 0.1
