"""GPU parity of the page2d rotary encoding (rswa_rope_page2d, rswa_append_rope) against
the oracle's fp64 rotation (oracle.rope_page2d).

Tolerance, from the kernel's arithmetic: it takes each angle in fp64, rounds cos and sin
to fp32 and forms x_i cos - x_{i+D/2} sin (and the partner) with one fp32 product and one
fp32 FMA. Each of those four roundings errs by at most 2^-24 of a term no larger than
|x_i| + |x_{i+D/2}|, so before its final rounding an output is within
E = 2^-22 (|x_i| + |x_{i+D/2}|) of the exact rotation (the fp64 angles differ from the
oracle's by ~1e-16 relative, negligible). Rounding to bf16 adds at most half a bf16 step
of the result. The test asserts |got - exact| <= E + half a step for every element, and
that at most 1 in 1000 elements differ from the correctly rounded value (oracle.bf16_round
of the exact rotation; the expected share is about 1e-4). The ring append around the
encoding is bit-exact (slot, wp, fill, untouched slots, the value row)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, assert_attention_close, to_np

pytestmark = pytest.mark.gpu


def _step(v: np.ndarray) -> np.ndarray:
    """Spacing of the bf16 grid at |v| (2^-133 at zero and in the subnormal range)."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, np.exp2(np.maximum(e - 7, -133)), 2.0 ** -133)


def assert_rope_close(got_bits: np.ndarray, x_bits: np.ndarray, tok, page, base, page_mod, what: str):
    """got_bits: the kernel's bf16 output for the bf16 input rows x_bits [..., H, D]."""
    exact = oracle.rope_page2d(x_bits, tok, page, base=base, page_mod=page_mod)
    assert got_bits.shape == exact.shape, what
    got = oracle.bf16_bits_to_f64(got_bits)
    x = np.abs(oracle.bf16_bits_to_f64(x_bits))
    h = x.shape[-1] // 2
    pair = x[..., :h] + x[..., h:]
    bound = 2.0 ** -22 * np.concatenate([pair, pair], axis=-1) + 0.5 * _step(got)
    err = np.abs(got - exact)
    worst = np.unravel_index(np.argmax(err - bound), err.shape)
    assert (err <= bound).all(), f"{what}: error {err[worst]:.3e} above bound {bound[worst]:.3e} at {worst}"
    off = int((got_bits != oracle.bf16_round(exact)).sum())
    assert off <= max(1, got_bits.size // 1000), f"{what}: {off} of {got_bits.size} not correctly rounded"


def _positions(rows, seed, neg=False):
    rng = np.random.default_rng(seed)
    tok = rng.integers(-50 if neg else 0, 20000, rows).astype(np.int32)
    page = rng.integers(-5 if neg else 0, 400, rows).astype(np.int32)
    return tok, page


@pytest.mark.parametrize("rows,H,D,page_mod,base", [
    (37, 3, 128, 2, 10000.0),      # ragged rows, one pass per row
    (5, 2, 16, 0, 10000.0),        # smallest head_dim, one axis
    (19, 5, 256, 3, 1e6),          # largest head_dim, page_mod 3
    (3, 128, 256, 1, 10000.0),     # 4096 chunk pairs per row: 16 passes, every pair on the page axis
    (300, 16, 128, 2, 500000.0),   # more rows than one CTA, grid-stride
])
def test_rope_page2d_matches_oracle(cuda_lib, rows, H, D, page_mod, base):
    g = synth._gen(900 + rows, "cuda")
    q = synth.randn_bf16((rows, H, D), g, "cuda", std=2.0)
    k = synth.randn_bf16((rows, H, D), g, "cuda")
    tok, page = _positions(rows, seed=rows, neg=True)
    q_out, k_out = torch.empty_like(q), torch.empty_like(k)
    cuda_lib.rswa_rope_page2d(q, torch.from_numpy(tok).cuda(), torch.from_numpy(page).cuda(), q_out=q_out, k=k,
                              k_out=k_out, base=base, page_mod=page_mod)
    torch.cuda.synchronize()
    assert_rope_close(to_np(q_out), to_np(q), tok, page, base, page_mod, "q")
    assert_rope_close(to_np(k_out), to_np(k), tok, page, base, page_mod, "k")


def test_rope_page2d_in_place_q_only_and_empty(cuda_lib):
    g = synth._gen(910, "cuda")
    x = synth.randn_bf16((4, 7, 9, 128), g, "cuda")          # leading dims [4][7] = 28 tokens
    tok, page = synth.page_positions(4, 7, seed=911)
    x_in = to_np(x).copy()
    cuda_lib.rswa_rope_page2d(x, tok.cuda(), page.cuda())    # in place, no k
    torch.cuda.synchronize()
    assert_rope_close(to_np(x), x_in, tok.numpy(), page.numpy(), 10000.0, 2, "in place")
    empty = torch.empty((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    z = torch.empty(0, dtype=torch.int32, device="cuda")
    cuda_lib.rswa_rope_page2d(empty, z, z)                    # nothing launched, no error


def test_rope_page2d_prefill_chunk_full_size(cuda_lib):
    # the benchmarked chunk: 4 sequences x 4096 tokens x 16 heads x 128 dims, q and k, every element
    B, T, H, D = 4, 4096, 16, 128
    g = synth._gen(920, "cuda")
    q = synth.randn_bf16((B, T, H, D), g, "cuda")
    k = synth.randn_bf16((B, T, H, D), g, "cuda")
    tok, page = synth.page_positions(B, T, seed=921)
    q_out, k_out = torch.empty_like(q), torch.empty_like(k)
    cuda_lib.rswa_rope_page2d(q, tok.cuda(), page.cuda(), q_out=q_out, k=k, k_out=k_out)
    torch.cuda.synchronize()
    assert_rope_close(to_np(q_out), to_np(q), tok.numpy(), page.numpy(), 10000.0, 2, "q chunk")
    assert_rope_close(to_np(k_out), to_np(k), tok.numpy(), page.numpy(), 10000.0, 2, "k chunk")


@pytest.mark.parametrize("B,H,n", [(6, 16, 128), (3, 20, 40), (2, 40, 7)])
def test_append_rope_matches_oracle(cuda_lib, B, H, n):
    g = synth._gen(930 + H, "cuda")
    ring_k = synth.randn_bf16((B, H, n, 128), g, "cuda")
    ring_v = synth.randn_bf16((B, H, n, 128), g, "cuda")
    k_new = synth.randn_bf16((B, H, 128), g, "cuda")
    v_new = synth.randn_bf16((B, H, 128), g, "cuda")
    q = synth.randn_bf16((B, H, 128), g, "cuda")
    rng = np.random.default_rng(H)
    wp = rng.integers(0, n, B).astype(np.int32)
    fill = rng.integers(0, n + 1, B).astype(np.int32)
    wp[-1] = -1                                                   # a bad ring state: flagged, ring untouched
    tok, page = _positions(B, seed=H + 1)
    o_rk, o_rv = to_np(ring_k).copy(), to_np(ring_v).copy()
    k_bits = to_np(k_new)
    # the ring holds the kernel's encoded key; the oracle's append takes the correctly rounded one
    want_k = oracle.bf16_round(oracle.rope_page2d(k_bits, tok, page))
    t_wp, t_fill = torch.from_numpy(wp).cuda(), torch.from_numpy(fill).cuda()
    slot = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(64, dtype=torch.int32, device="cuda")
    q_out = torch.empty_like(q)
    cuda_lib.rswa_append_rope(ring_k, ring_v, k_new, v_new, t_wp, t_fill, q, torch.from_numpy(tok).cuda(),
                              torch.from_numpy(page).cuda(), q_out=q_out, slot_out=slot, status=status)
    assert cuda_lib.check_status(status) == 0x2                     # RSWA_DEVICE_BAD_RING_STATE
    assert_rope_close(to_np(q_out), to_np(q), tok, page, 10000.0, 2, "q_out")
    # the oracle's append of the encoded key for the sequences with a valid ring
    ok = slice(0, B - 1)
    o_wp, o_fill = wp[ok].copy(), fill[ok].copy()
    o_rk_ok, o_rv_ok = o_rk[ok].copy(), o_rv[ok].copy()
    o_slot = oracle.append(o_rk_ok, o_rv_ok, want_k[ok], to_np(v_new)[ok], o_wp, o_fill)
    np.testing.assert_array_equal(to_np(slot)[ok], o_slot)
    np.testing.assert_array_equal(to_np(t_wp)[ok], o_wp)
    np.testing.assert_array_equal(to_np(t_fill)[ok], o_fill)
    got_rk, got_rv = to_np(ring_k), to_np(ring_v)
    for b in range(B - 1):
        s = o_slot[b]
        assert_rope_close(got_rk[b, :, s][None], k_bits[b][None], tok[b:b + 1], page[b:b + 1], 10000.0, 2,
                          f"ring_k slot b={b}")
        others = np.arange(n) != s
        np.testing.assert_array_equal(got_rk[b][:, others], o_rk_ok[b][:, others])
        np.testing.assert_array_equal(got_rv[b], o_rv_ok[b])
    # the flagged sequence: ring, wp, fill and slot_out untouched
    np.testing.assert_array_equal(got_rk[-1], o_rk[-1])
    np.testing.assert_array_equal(got_rv[-1], o_rv[-1])
    assert to_np(t_wp)[-1] == -1 and to_np(t_fill)[-1] == fill[-1] and to_np(slot)[-1] == -7


def test_srswa_step_with_page2d_encoding(cuda_lib):
    # rswa_append_rope + srswa_decode on the encoded query against the oracle's encoding,
    # append and SR-SWA decode, over several steps that cross a page boundary
    plen = [32 * 40, 32 * 33 + 5, 32 * 20]
    B, H, n, steps = 3, 16, 128, 6
    case = synth.decode_case(B, H, 128, plen, 32 * 40, n, steps, seed=940, device="cuda", fill0=[128, 50, 0])
    tok, page = synth.page_positions(B, steps, seed=941, page_len=(2, 4))
    ring_k, ring_v, wp, fill = case.ring_k.clone(), case.ring_v.clone(), case.wp.clone(), case.fill.clone()
    dims = cuda_lib.dims_of(case.pk, case.ring_k)
    ws = cuda_lib.new_workspace(dims, cuda_lib.OP_SRSWA_DECODE)
    out = torch.empty((B, H, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    q_rot = torch.empty((B, H, 128), dtype=torch.bfloat16, device="cuda")
    o_rk, o_rv, o_wp, o_fill = to_np(ring_k).copy(), to_np(ring_v).copy(), to_np(wp).copy(), to_np(fill).copy()
    rng = np.random.default_rng(942)
    for s in range(steps):
        t_s, p_s = tok[:, s].contiguous(), page[:, s].contiguous()
        cuda_lib.rswa_append_rope(ring_k, ring_v, case.k_new[s], case.v_new[s], wp, fill, case.q[s], t_s.cuda(),
                                  p_s.cuda(), q_out=q_rot, status=ws)
        blk = np.stack([rng.permutation((m + 31) // 32)[:16] for m in plen]).astype(np.int32)
        logp = np.log(rng.dirichlet(np.ones(16), B)).astype(np.float32)
        cuda_lib.srswa_decode(q_rot, case.pk, case.pv, case.prefix_len, torch.from_numpy(blk).cuda(),
                              torch.from_numpy(logp).cuda(), ring_k, ring_v, wp, fill, out, ws, lse=lse,
                              scale=case.scale)
        qo = oracle.bf16_round(oracle.rope_page2d(to_np(case.q[s]), t_s.numpy(), p_s.numpy()))
        ko = oracle.bf16_round(oracle.rope_page2d(to_np(case.k_new[s]), t_s.numpy(), p_s.numpy()))
        oracle.append(o_rk, o_rv, ko, to_np(case.v_new[s]), o_wp, o_fill)
        ref, ref_lse = oracle.srswa_decode(qo, to_np(case.pk), to_np(case.pv), to_np(case.prefix_len), blk,
                                           logp.astype(np.float64), o_rk, o_rv, o_wp, o_fill, case.scale)
        assert_attention_close(to_np(out), ref, f"page2d SR-SWA step {s}")
        assert np.abs(to_np(lse) - ref_lse).max() <= LSE_ABS
    assert cuda_lib.check_status(ws) == 0
