"""GPU parity of the per-token router of the chunked prefill (srswa_route_tokens) over the
paths its kernel takes for histories of at most 1024 blocks, against the oracle's router
taken row by row:
* planted routes (16 candidates: the sort-based threshold): indices bit-exact, p within 1e-5,
  and the same routes as the decode router (srswa_route) called token by token;
* fewer candidates than top-k (the rest of the top-k by argmax rounds), with ties (equal
  scores rank by the smaller block) and histories shorter than k blocks: indices bit-exact;
* more than 32 candidates (threshold by bisection and the closed form over the support):
  p within 1e-5, and the selection a valid top-k (random scores may hold near-ties);
* an empty history and a bad prefix length (flagged, no blocks); odd token counts, a single
  sequence spread over many CTAs.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import ROUTER_P_ABS, to_np

pytestmark = pytest.mark.gpu


def _run(rswa, q_tok, kbar, plen, cap, topk=16, check=True):
    B, T, _ = q_tok.shape
    blk = torch.full((B, T, topk), -7, dtype=torch.int32, device="cuda")
    logp = torch.full((B, T, topk), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    rswa.srswa_route_tokens(q_tok, kbar, torch.tensor(plen, dtype=torch.int32, device="cuda"), blk, logp, ws,
                            prefix_cap=cap)
    status = rswa.check_status(ws)
    if check:
        assert status == 0
    return to_np(blk), to_np(logp), status


def _oracle_rows(q_tok, kbar, plen, topk=16):
    """oracle.route over the B * T rows (each token's row against its sequence's keys)."""
    q_tok, kbar = np.asarray(q_tok, np.float32), np.asarray(kbar, np.float64)
    B, T, DI = q_tok.shape
    r = oracle.route(q_tok.reshape(B * T, DI), np.repeat(kbar, T, axis=0), np.repeat(np.asarray(plen, np.int32), T),
                     topk=topk)
    return {k: (v.reshape((B, T) + v.shape[1:]) if isinstance(v, np.ndarray) and v.ndim >= 1 else v)
            for k, v in r.items()}


@pytest.mark.parametrize("plen,T", [
    ([32 * 1024, 32 * 700 + 5, 32 * 64], 101),   # full, ragged and short histories; odd T
    ([32 * 1024], 4096),                         # one sequence over every SM, 28 tokens per CTA
])
def test_route_tokens_planted(cuda_lib, plen, T):
    cap = max(plen)
    B = len(plen)
    pl = synth.plant_router_keys(plen, cap, n_dirs=32, seed=1201 + T, device="cuda")
    dirs = torch.arange(T, device="cuda") % 32
    q_tok = pl.q_idx[dirs].permute(1, 0, 2).contiguous()
    pt = torch.tensor(plen, dtype=torch.int32, device="cuda")
    kbar = torch.empty((B, (cap + 31) // 32, 32), dtype=torch.float32, device="cuda")
    cuda_lib.srswa_index_pool(pl.k_idx, pt, kbar)
    blk, logp, _ = _run(cuda_lib, q_tok, kbar, plen, cap)
    o_kbar = oracle.index_pool(to_np(pl.k_idx), np.array(plen, np.int32))
    rows = np.arange(T) if T <= 128 else np.sort(np.random.default_rng(3).choice(T, 96, replace=False))
    r_idx, r_logp = oracle.route_tokens(to_np(q_tok)[:, rows], o_kbar, np.array(plen, np.int32))
    np.testing.assert_array_equal(blk[:, rows], r_idx)
    np.testing.assert_allclose(np.exp(logp[:, rows]), np.exp(r_logp), rtol=0, atol=ROUTER_P_ABS)
    np.testing.assert_array_equal(blk[:, rows], to_np(pl.planted)[rows % 32].transpose(1, 0, 2))
    # the decode router on the same rows, one token at a time: the same blocks, p within 1e-6
    d_blk = torch.empty((B, 16), dtype=torch.int32, device="cuda")
    d_logp = torch.empty((B, 16), dtype=torch.float32, device="cuda")
    ws = cuda_lib.route_workspace(B, cap)
    for t in rows[:24]:
        cuda_lib.srswa_route(q_tok[:, t].contiguous(), kbar, pt, d_blk, d_logp, ws, prefix_cap=cap)
        np.testing.assert_array_equal(blk[:, t], to_np(d_blk))
        np.testing.assert_allclose(np.exp(logp[:, t]), np.exp(to_np(d_logp)), rtol=0, atol=1e-6)


def test_route_tokens_fewer_candidates_than_topk_ties_and_short_histories(cuda_lib):
    # q = e0 and scores kbar[., c, 0]: one block far above the rest (a single entmax candidate),
    # the rest of the top-16 by argmax rounds, with equal scores ranked by the smaller block
    nb_cap, T = 300, 5
    rng = np.random.default_rng(1301)
    kbar = np.zeros((3, nb_cap, 32), np.float32)
    for b in range(3):
        vals = rng.permutation(np.arange(nb_cap, dtype=np.float32) * 0.02)   # distinct, gaps 0.02, below 6
        vals[[7, 19, 40, 41, 250]] = 7.0                                     # a five-way tie behind the top
        vals[123] = 12.0                                                     # the only candidate (cut: 10)
        kbar[b, :, 0] = vals
    q = np.zeros((3, T, 32), np.float32)
    q[:, :, 0] = 1.0
    q[:, 1, 0] = 0.5                                                         # other scales: the same order
    plen = [nb_cap * 32, 200 * 32 + 7, 3 * 32 - 4]                           # the last: 3 blocks < 16
    blk, logp, _ = _run(cuda_lib, torch.from_numpy(q).cuda(), torch.from_numpy(kbar).cuda(), plen, nb_cap * 32)
    r = _oracle_rows(q, kbar, plen)
    np.testing.assert_array_equal(blk, r["blk_idx"])
    np.testing.assert_allclose(np.exp(logp), np.exp(r["blk_logp"]), rtol=0, atol=ROUTER_P_ABS)
    assert (blk[0, 0, :6] == [123, 7, 19, 40, 41, 250]).all()               # the tie in block order
    assert (blk[2, :, 3:] == -1).all() and np.isneginf(logp[2, :, 3:]).all()


@pytest.mark.parametrize("seed,nb,spread", [(11, 1000, 0.02), (12, 700, 0.2), (13, 64, 1.0), (14, 1024, 0.05)])
def test_route_tokens_many_candidates(cuda_lib, seed, nb, spread):
    # unplanted scores: up to every block a candidate (the bisection path); near-ties possible
    rng = np.random.default_rng(seed)
    B, T = 2, 9
    kbar = rng.normal(0, spread, (B, nb, 32)).astype(np.float32)
    q = rng.normal(0, 1, (B, T, 32)).astype(np.float32)
    plen = [nb * 32, nb * 16 + 3]
    blk, logp, _ = _run(cuda_lib, torch.from_numpy(q).cuda(), torch.from_numpy(kbar).cuda(), plen, nb * 32)
    r = _oracle_rows(q, kbar, plen)
    for b in range(B):
        nbb = (plen[b] + 31) // 32
        for t in range(T):
            z = r["z"][b, t]
            got = blk[b, t]
            assert len(set(got.tolist())) == 16 and (got >= 0).all() and (got < nbb).all()
            np.testing.assert_allclose(np.sort(z[got])[::-1], np.sort(z[:nbb])[::-1][:16], rtol=0, atol=1e-5)
            assert (np.diff(z[got]) <= 1e-5).all()                            # descending
            np.testing.assert_allclose(np.exp(logp[b, t]), r["probs"][b, t][got], rtol=0, atol=ROUTER_P_ABS)
    # candidates (z > max z - 2) per row: spread <= 0.05 puts every row on the bisection path,
    # spread 0.2 rows on both paths
    n_c = np.concatenate([(zz > zz.max(axis=-1, keepdims=True) - 2).sum(axis=-1)
                          for zz in (r["z"][b, :, :(plen[b] + 31) // 32] for b in range(B))])
    if spread <= 0.05:
        assert (n_c > 32).all()
    elif spread == 0.2:
        assert (n_c > 32).any() and (n_c <= 32).any()


def test_route_tokens_empty_and_bad_histories(cuda_lib):
    rng = np.random.default_rng(1401)
    nb_cap, T = 40, 4
    kbar = rng.normal(0, 1, (3, nb_cap, 32)).astype(np.float32)
    q = rng.normal(0, 1, (3, T, 32)).astype(np.float32)
    plen = [0, nb_cap * 32, -5]                                              # empty, full, bad
    blk, logp, status = _run(cuda_lib, torch.from_numpy(q).cuda(), torch.from_numpy(kbar).cuda(), plen,
                             nb_cap * 32, check=False)
    assert status == cuda_lib.binding.DEVICE_BAD_PREFIX_LEN
    for b in (0, 2):
        assert (blk[b] == -1).all() and np.isneginf(logp[b]).all()
    r = _oracle_rows(q[1:2], kbar[1:2], plen[1:2])
    np.testing.assert_allclose(np.exp(logp[1]), np.exp(r["blk_logp"][0]), rtol=0, atol=ROUTER_P_ABS)
