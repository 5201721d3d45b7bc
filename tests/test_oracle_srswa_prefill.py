"""Pins of the oracle's SR-SWA chunked prefill.

- per-token routes: with planted router keys every token recovers its planted
  top-16 in order (the construction of synth.plant_router_keys).
- prefill row i equals the SR-SWA decode (oracle_srswa_decode, separately pinned)
  after appending outputs 0..i to an empty ring, with row i's route: the band
  logic of the prefill against the ring logic of the decode.
- every block routed with zero bias equals the R-SWA prefill (pinned against
  an explicit-mask brute force).
- a chunk run as two chunks, the second reading the first's last n outputs
  through the ring, equals the single chunk.
"""
import numpy as np
import torch

import oracle
from long_context_decode_swa_b200 import synth


def _case(B, H, plen, cap, T, seed):
    d = synth.prefill_case(B, H, 128, plen, cap, T, seed=seed, poison=False)
    return {k: (synth.to_u16(v) if torch.is_tensor(v) and v.dtype == torch.bfloat16 else v) for k, v in d.items()}


def test_route_tokens_recovers_planted_blocks():
    plen, cap, T = [32 * 40, 32 * 23 + 5], 32 * 40, 6
    pl = synth.plant_router_keys(plen, cap, n_dirs=T, seed=31)
    kbar = oracle.index_pool(synth.to_u16(pl.k_idx), np.array(plen, np.int32))
    q_tok = pl.q_idx.numpy().transpose(1, 0, 2).copy()               # token t uses direction t: [B][T][32]
    blk, logp = oracle.route_tokens(q_tok, kbar, np.array(plen, np.int32))
    np.testing.assert_array_equal(blk, pl.planted.numpy().transpose(1, 0, 2))
    assert np.isfinite(logp).all()


def test_prefill_rows_equal_sequential_decode():
    B, H, n, T = 2, 2, 16, 24
    plen, cap = np.array([200, 77], np.int32), 200
    d = _case(B, H, plen, cap, T, 41)
    rng = np.random.default_rng(4)
    blk = np.stack([np.stack([rng.permutation((m + 31) // 32)[:3] for _ in range(T)]) for m in plen]).astype(np.int32)
    logp = np.log(rng.dirichlet(np.ones(3), size=(B, T)))
    blk[1, 3, 2] = -1
    logp[0, 5, 1] = -np.inf
    rows = np.arange(T)
    out, lse = oracle.srswa_prefill(d["q"], d["k_out"], d["v_out"], d["pk"], d["pv"], plen, blk, logp, d["scale"],
                                    rows, n)
    rk = np.zeros((B, H, n, 128), np.uint16)
    rv = np.zeros_like(rk)
    wp = np.zeros(B, np.int32)
    fill = np.zeros(B, np.int32)
    for i in range(T):
        oracle.append(rk, rv, np.ascontiguousarray(d["k_out"][:, :, i]), np.ascontiguousarray(d["v_out"][:, :, i]),
                      wp, fill)
        ref, ref_lse = oracle.srswa_decode(np.ascontiguousarray(d["q"][:, :, i]), d["pk"], d["pv"], plen,
                                           blk[:, i], logp[:, i], rk, rv, wp.copy(), fill.copy(), d["scale"])
        np.testing.assert_allclose(out[:, :, i], ref, rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], ref_lse, rtol=1e-12, atol=1e-12)


def test_all_blocks_zero_bias_equals_rswa_prefill():
    B, H, n, T = 2, 2, 8, 20
    plen, cap = np.array([96, 50], np.int32), 96
    d = _case(B, H, plen, cap, T, 42)
    nb = 3
    blk = np.tile(np.arange(nb, dtype=np.int32), (B, T, 1))
    blk[1, :, 2] = -1                                                  # sequence 1 has only 2 blocks
    logp = np.zeros((B, T, nb))
    rows = np.arange(T)
    got, got_lse = oracle.srswa_prefill(d["q"], d["k_out"], d["v_out"], d["pk"], d["pv"], plen, blk, logp,
                                        d["scale"], rows, n)
    ref, ref_lse = oracle.rswa_prefill(d["q"], d["k_out"], d["v_out"], d["pk"], d["pv"], plen, d["scale"], rows, n)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(got_lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_two_chunks_through_the_ring_equal_one_chunk():
    B, H, n, T = 1, 2, 8, 20
    plen, cap = np.array([64], np.int32), 64
    d = _case(B, H, plen, cap, T, 43)
    rng = np.random.default_rng(5)
    blk = np.stack([rng.permutation(2)[None].repeat(T, 0)]).astype(np.int32)   # [1][T][2]
    logp = np.log(np.full((B, T, 2), 0.5))
    one, _ = oracle.srswa_prefill(d["q"], d["k_out"], d["v_out"], d["pk"], d["pv"], plen, blk, logp, d["scale"],
                                  np.arange(T), n)
    h = 12                                                            # second chunk: outputs 12..19
    ring_k = np.zeros((B, H, n, 128), np.uint16)
    ring_v = np.zeros_like(ring_k)
    wp = np.zeros(B, np.int32)
    fill = np.zeros(B, np.int32)
    for i in range(h):
        oracle.append(ring_k, ring_v, np.ascontiguousarray(d["k_out"][:, :, i]),
                      np.ascontiguousarray(d["v_out"][:, :, i]), wp, fill)
    sub = {k: np.ascontiguousarray(d[k][:, :, h:]) for k in ("q", "k_out", "v_out")}
    two, _ = oracle.srswa_prefill(sub["q"], sub["k_out"], sub["v_out"], d["pk"], d["pv"], plen,
                                  np.ascontiguousarray(blk[:, h:]), np.ascontiguousarray(logp[:, h:]), d["scale"],
                                  np.arange(T - h), n, ring_k=ring_k, ring_v=ring_v, wp=wp, fill=fill)
    np.testing.assert_allclose(two, one[:, :, h:], rtol=1e-12, atol=1e-13)
