"""Pins of the oracle's page2d rotary encoding and of its bf16 rounding.

The pages name the two axes of the encoding (Unlimited-OCR-2 SR-SWA explainer,
2D 位置编码: an in-page token axis and a page axis, page_mod 2) but not its
constants; the oracle's readings are the LLaMA family's half-split pairs and
frequencies base^(-2i/D), with page_mod interleaving the pairs between the axes.
The pins tie those readings to an implementation the oracle does not share:

- page_mod 0 (one axis) equals the LLaMA rotary routine of the transformers
  library (LlamaRotaryEmbedding + apply_rotary_pos_emb) at the token position;
  so does page_mod 2 when the page number equals the token position;
- axis separation: page 0 leaves the page-axis pairs bit-for-bit unchanged and
  the token-axis pairs equal the library's encoding at the token position;
  token position 0 does the converse; page_mod 3 moves pairs 2, 5, 8, ...;
- relative position: q.k after the encoding depends only on the differences of
  the two tokens' positions on each axis; every pair keeps its norm;
- bf16 rounding equals torch's float32 -> bfloat16 conversion (round to
  nearest even) on float32-representable values, with the tie cases by hand.

A dropped term, a sign, a frequency index, a pairing or an axis assignment off
fails one of these.
"""
import numpy as np
import pytest
import torch

import oracle

D = 128


def _bf16(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return oracle.bf16_round(rng.standard_normal(shape) * scale)


@pytest.fixture(scope="module")
def library_rope():
    """The transformers LLaMA rotary encoding of bf16 rows x [R][H][D] at positions pos [R]."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaRotaryEmbedding, apply_rotary_pos_emb

    def run(x_bits, pos, base=10000.0):
        H = x_bits.shape[1]
        cfg = LlamaConfig(hidden_size=H * D, num_attention_heads=H, num_key_value_heads=H, head_dim=D,
                          rope_theta=base, max_position_embeddings=1 << 16)
        emb = LlamaRotaryEmbedding(cfg)
        x = torch.from_numpy(oracle.bf16_bits_to_f64(x_bits)).permute(1, 0, 2).unsqueeze(0)  # [1][H][R][D]
        cos, sin = emb(x, torch.from_numpy(np.asarray(pos, np.int64)).unsqueeze(0))
        y, _ = apply_rotary_pos_emb(x, x, cos.to(torch.float64), sin.to(torch.float64))
        return y.squeeze(0).permute(1, 0, 2).numpy()

    return run


# the library takes its angles in float32: at positions below 2048 an angle is off by at most
# about 2048 * 2^-23 rad, so an element of magnitude below 5 moves by well under 2e-3
LIB_ATOL = 2e-3


@pytest.mark.parametrize("base", [10000.0, 1e6])
def test_one_axis_equals_library(library_rope, base):
    x = _bf16((24, 4, D), seed=1)
    pos = np.random.default_rng(2).integers(0, 2048, 24).astype(np.int32)
    got = oracle.rope_page2d(x, pos, np.zeros(24, np.int32), base=base, page_mod=0)
    np.testing.assert_allclose(got, library_rope(x, pos, base), rtol=0, atol=LIB_ATOL)


def test_equal_axes_equal_library(library_rope):
    x = _bf16((16, 3, D), seed=3)
    pos = np.random.default_rng(4).integers(0, 2048, 16).astype(np.int32)
    got = oracle.rope_page2d(x, pos, pos, page_mod=2)
    np.testing.assert_allclose(got, library_rope(x, pos), rtol=0, atol=LIB_ATOL)


def _pair_dims(pairs):
    pairs = np.asarray(pairs)
    return np.concatenate([pairs, pairs + D // 2])


def test_axis_separation(library_rope):
    x = _bf16((12, 2, D), seed=5)
    x64 = oracle.bf16_bits_to_f64(x)
    rng = np.random.default_rng(6)
    tok = rng.integers(1, 2048, 12).astype(np.int32)
    pg = rng.integers(1, 400, 12).astype(np.int32)
    zero = np.zeros(12, np.int32)
    even, odd = _pair_dims(np.arange(0, D // 2, 2)), _pair_dims(np.arange(1, D // 2, 2))

    on_tok = oracle.rope_page2d(x, tok, zero, page_mod=2)          # page 0: page-axis (odd) pairs untouched
    assert np.array_equal(on_tok[..., odd], x64[..., odd])
    np.testing.assert_allclose(on_tok[..., even], library_rope(x, tok)[..., even], rtol=0, atol=LIB_ATOL)

    on_page = oracle.rope_page2d(x, zero, pg, page_mod=2)          # token 0: token-axis (even) pairs untouched
    assert np.array_equal(on_page[..., even], x64[..., even])
    np.testing.assert_allclose(on_page[..., odd], library_rope(x, pg)[..., odd], rtol=0, atol=LIB_ATOL)

    third = _pair_dims(np.arange(2, D // 2, 3))                     # page_mod 3: pairs 2, 5, 8, ... on the page axis
    rest = np.setdiff1d(np.arange(D), third)
    got = oracle.rope_page2d(x, zero, pg, page_mod=3)
    assert np.array_equal(got[..., rest], x64[..., rest])
    np.testing.assert_allclose(got[..., third], library_rope(x, pg)[..., third], rtol=0, atol=LIB_ATOL)

    every = oracle.rope_page2d(x, zero, pg, page_mod=1)             # page_mod 1: every pair on the page axis
    np.testing.assert_allclose(every, library_rope(x, pg), rtol=0, atol=LIB_ATOL)


def test_relative_position_invariance():
    rng = np.random.default_rng(7)
    R, H = 40, 4
    q, k = _bf16((R, H, D), seed=8), _bf16((R, H, D), seed=9)
    t1, t2 = rng.integers(0, 20000, R).astype(np.int32), rng.integers(0, 20000, R).astype(np.int32)
    p1, p2 = rng.integers(0, 400, R).astype(np.int32), rng.integers(0, 400, R).astype(np.int32)
    s, u = rng.integers(-5000, 5000, R).astype(np.int32), rng.integers(-300, 300, R).astype(np.int32)

    def dots(a, b, c, d):
        return np.einsum("rhd,rhd->rh", oracle.rope_page2d(q, a, b), oracle.rope_page2d(k, c, d))

    base = dots(t1, p1, t2, p2)
    np.testing.assert_allclose(dots(t1 + s, p1 + u, t2 + s, p2 + u), base, rtol=0, atol=1e-9)
    # and it does depend on each axis's difference
    assert np.abs(dots(t1 + 1, p1, t2, p2) - base).max() > 1e-3
    assert np.abs(dots(t1, p1 + 1, t2, p2) - base).max() > 1e-3


def test_pair_norms_preserved():
    x = _bf16((20, 3, D), seed=10)
    rng = np.random.default_rng(11)
    got = oracle.rope_page2d(x, rng.integers(0, 20000, 20).astype(np.int32),
                             rng.integers(0, 400, 20).astype(np.int32))
    x64 = oracle.bf16_bits_to_f64(x)
    h = D // 2
    np.testing.assert_allclose(got[..., :h] ** 2 + got[..., h:] ** 2, x64[..., :h] ** 2 + x64[..., h:] ** 2,
                               rtol=1e-12, atol=1e-14)


def test_bf16_round_matches_torch():
    rng = np.random.default_rng(12)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        (rng.standard_normal(20000) * np.exp2(rng.integers(-140, 120, 20000))).astype(np.float32),
                        np.float32([0.0, -0.0, 1.0, -3.0, 3.38e38, 1e-45, -2.5e-41])])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_round(v.astype(np.float64)), want)


def test_bf16_round_ties_and_round_trips():
    got = oracle.bf16_round(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8), 2.0 ** -133 * 1.5]))
    assert got.tolist() == [0x3F80, 0x3F82, 0xBF80, 0x0002]
    bits = np.arange(0, 0x7F80, 7, dtype=np.uint16)                   # finite non-negative patterns
    assert np.array_equal(oracle.bf16_round(oracle.bf16_bits_to_f64(bits)), bits)
