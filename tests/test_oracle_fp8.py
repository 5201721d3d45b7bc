"""Pins of the oracle's FP8 (E4M3) prefix: codec, quantiser and the FP8 decodes.

- codec: the E4M3 format's definition (bias 7, 3 mantissa bits, subnormals
  m/8 * 2^-6, S.1111.111 = NaN, largest finite 448) fixes landmark codes; every
  finite code survives a round trip; the encoder is checked against an
  exhaustive nearest-value search over the 254 finite values (ties to the even
  mantissa, saturation at 448), which shares nothing with it.
- quantiser: per (sequence, head, 32-token block) scale = amax / 448 in fp32;
  the block's largest element lands on +-448; every element is within half a
  grid step of its dequantised value; rows past the prefix are zero codes.
- FP8 decodes: data on the E4M3 grid with a 448 in every block, each block then
  times its own power of two (small enough that the softmax is not saturated),
  get exactly that power of two as scale, so the FP8 decode must equal the
  (pinned) bf16 decode of the same values exactly, for R-SWA and for SR-SWA.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth


def _table():
    return oracle.e4m3_to_double(np.arange(256, dtype=np.uint8))


def test_e4m3_landmarks():
    t = _table()
    assert t[0x00] == 0.0 and np.signbit(t[0x80])
    assert t[0x01] == 2.0 ** -9 and t[0x07] == 7 * 2.0 ** -9        # subnormals m/8 * 2^-6
    assert t[0x08] == 2.0 ** -6                                     # smallest normal
    assert t[0x38] == 1.0 and t[0x39] == 1.125 and t[0x30] == 0.5
    assert t[0x7e] == 448.0 and t[0xfe] == -448.0                   # largest finite
    assert np.isnan(t[0x7f]) and np.isnan(t[0xff])                  # the only NaNs
    assert np.isfinite(np.delete(t, [0x7f, 0xff])).all()
    pos = t[:0x7f]
    assert (np.diff(pos) > 0).all()                                 # codes 0..0x7e increase


def test_e4m3_round_trip_every_finite_code():
    t = _table()
    codes = np.array([c for c in range(256) if c not in (0x7f, 0xff)], np.uint8)
    back = oracle.e4m3_encode(t[codes].astype(np.float32))
    np.testing.assert_array_equal(back, codes)


def _nearest_code(x: float, t: np.ndarray) -> int:
    """Exhaustive search: the finite code nearest to x, ties to the even code (even mantissa)."""
    if abs(x) >= 448.0:
        return 0x7e | (0x80 if x < 0 else 0)
    finite = [c for c in range(0x7f)]                     # non-negative finite codes
    a = abs(x)
    d = np.array([abs(t[c] - a) for c in finite])
    best = np.flatnonzero(d == d.min())
    c = finite[best[0]] if len(best) == 1 else [finite[i] for i in best if finite[i] % 2 == 0][0]
    return c | (0x80 if np.signbit(x) else 0)


def test_e4m3_encoder_against_exhaustive_search():
    t = _table()
    rng = np.random.default_rng(11)
    mags = np.exp2(rng.uniform(-12, 9.5, 3000))
    xs = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    pos = t[:0x7f]
    mids = ((pos[:-1] + pos[1:]) / 2).astype(np.float32)                # every tie, exactly representable
    xs = np.concatenate([xs, mids, -mids, np.float32([0.0, 447.9, 448.0, 463.9, 464.0, 1e9, 2.0 ** -10])])
    got = oracle.e4m3_encode(xs)
    want = np.array([_nearest_code(float(x), t) for x in xs], np.uint8)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("plen", [[200, 64], [31, 1]])
def test_quantize_prefix_properties(plen):
    B, H, cap, D = 2, 3, 224, 128
    g = torch.Generator().manual_seed(5)
    x = (torch.randn((B, H, cap, D), generator=g) * torch.exp(torch.randn((B, H, cap, 1), generator=g))).bfloat16()
    xu = synth.to_u16(x)
    xf = x.float().numpy().astype(np.float64)
    codes, scales = oracle.quantize_prefix(xu, np.array(plen, np.int32))
    t = _table()
    deq_unit = t[codes]
    for b, m in enumerate(plen):
        for h in range(H):
            for c in range((m + 31) // 32):
                rows = slice(32 * c, min(m, 32 * c + 32))
                blk = xf[b, h, rows]
                amax = np.float32(np.abs(blk).max())
                assert scales[b, h, c] == np.float32(amax / np.float32(448.0))
                deq = deq_unit[b, h, rows] * float(scales[b, h, c])
                # the block maximum maps onto +-448 (up to the fp32 rounding of the scale)
                assert np.isclose(np.abs(deq).max(), amax, rtol=2 ** -20)
                # within half a grid step: 2^-4 relative for normals, 2^-10 * scale absolute below
                err = np.abs(deq - blk)
                bound = np.maximum(np.abs(blk) * 2.0 ** -4, 2.0 ** -10 * float(scales[b, h, c])) * (1 + 2 ** -20)
                assert (err <= bound).all()
            tail = slice(m, min(cap, 32 * ((m + 31) // 32)))
            assert (codes[b, h, tail] == 0).all()
            assert (scales[b, h, (m + 31) // 32:] == 0).all()


GRID_POW2 = (-10, -6)   # block / row factors 2^e: keeps q.k moderate, so the softmax is not saturated


def _grid_prefix(B, H, cap, D, seed):
    """bf16 prefix on the E4M3 grid with a 448 in every 32-row block, each block then times its
    own 2^e, e in GRID_POW2: every block scale is exactly 2^e and every element exactly its
    code value times that scale. Returns (prefix, e [B][H][blocks])."""
    rng = np.random.default_rng(seed)
    t = _table()
    sign = (rng.integers(0, 2, (B, H, cap, D)) << 7).astype(np.uint8)
    codes = rng.integers(0, 0x7f, (B, H, cap, D)).astype(np.uint8) | sign   # finite codes only
    codes[:, :, ::32, 0] = 0x7e                                             # amax = 448 in every block
    e = rng.integers(GRID_POW2[0], GRID_POW2[1] + 1, (B, H, (cap + 31) // 32))
    f = np.repeat(np.exp2(e), 32, axis=2)[:, :, :cap, None]
    return torch.from_numpy((t[codes] * f).astype(np.float32)).bfloat16(), e   # exact: E4M3 x 2^e fits bf16


def _check_grid_scales(scales, e, plen):
    for b, m in enumerate(plen):
        nb = (m + 31) // 32
        np.testing.assert_array_equal(scales[b, :, :nb], np.exp2(e[b, :, :nb]).astype(np.float32))


def test_rswa_decode_fp8_equals_bf16_on_grid_data():
    B, H, D, n, cap = 2, 2, 128, 8, 96
    c = synth.decode_case(B, H, D, [96, 70], cap, n, 1, seed=21, wp0=3, fill0=8)
    pk, ek = _grid_prefix(B, H, cap, D, 1)
    pv, ev = _grid_prefix(B, H, cap, D, 2)
    plen = c.prefix_len.numpy()
    k8, ks = oracle.quantize_prefix(synth.to_u16(pk), plen)
    v8, vs = oracle.quantize_prefix(synth.to_u16(pv), plen)
    _check_grid_scales(ks, ek, plen)
    _check_grid_scales(vs, ev, plen)
    args = (synth.to_u16(c.ring_k), synth.to_u16(c.ring_v), c.wp.numpy(), c.fill.numpy(), c.scale)
    ref, ref_lse = oracle.rswa_decode(synth.to_u16(c.q[0]), synth.to_u16(pk), synth.to_u16(pv), plen, *args)
    got, got_lse = oracle.rswa_decode_fp8(synth.to_u16(c.q[0]), k8, v8, ks, vs, plen, *args)
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(got_lse, ref_lse)


def test_srswa_decode_fp8_equals_bf16_on_grid_data():
    B, H, D, n, cap = 2, 2, 128, 8, 160
    c = synth.decode_case(B, H, D, [160, 100], cap, n, 1, seed=22, wp0=5, fill0=8)
    pk, ek = _grid_prefix(B, H, cap, D, 3)
    pv, ev = _grid_prefix(B, H, cap, D, 4)
    plen = c.prefix_len.numpy()
    k8, ks = oracle.quantize_prefix(synth.to_u16(pk), plen)
    v8, vs = oracle.quantize_prefix(synth.to_u16(pv), plen)
    _check_grid_scales(ks, ek, plen)
    _check_grid_scales(vs, ev, plen)
    blk = np.array([[4, 0, 2, -1], [3, 1, 0, 2]], np.int32)
    logp = np.log(np.array([[0.5, 0.3, 0.2, 1.0], [0.4, 0.3, 0.2, 0.1]]))
    args = (synth.to_u16(c.ring_k), synth.to_u16(c.ring_v), c.wp.numpy(), c.fill.numpy(), c.scale)
    ref, ref_lse = oracle.srswa_decode(synth.to_u16(c.q[0]), synth.to_u16(pk), synth.to_u16(pv), plen, blk, logp,
                                       *args)
    got, got_lse = oracle.srswa_decode_fp8(synth.to_u16(c.q[0]), k8, v8, ks, vs, plen, blk, logp, *args)
    np.testing.assert_array_equal(got, ref)
    np.testing.assert_array_equal(got_lse, ref_lse)


def test_fp8_decode_tracks_bf16_decode_on_gaussian_data():
    # quantisation error only: relative L2 of a few percent at most for N(0,1) data
    B, H, D, n, cap = 2, 2, 128, 16, 256
    c = synth.decode_case(B, H, D, [256, 190], cap, n, 1, seed=23, wp0=0, fill0=16)
    plen = c.prefix_len.numpy()
    k8, ks = oracle.quantize_prefix(synth.to_u16(c.pk), plen)
    v8, vs = oracle.quantize_prefix(synth.to_u16(c.pv), plen)
    args = (synth.to_u16(c.ring_k), synth.to_u16(c.ring_v), c.wp.numpy(), c.fill.numpy(), c.scale)
    ref, _ = oracle.rswa_decode(synth.to_u16(c.q[0]), synth.to_u16(c.pk), synth.to_u16(c.pv), plen, *args)
    got, _ = oracle.rswa_decode_fp8(synth.to_u16(c.q[0]), k8, v8, ks, vs, plen, *args)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert 0 < rel < 0.1
