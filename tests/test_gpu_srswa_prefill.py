"""GPU parity of the SR-SWA chunked prefill (per-token router; band part and routed part on
the tensor cores, merged by log-sum-exp) against the oracle.

Routes: block indices bit-exact, probabilities within 1e-5 (planted keys keep every
decisive score gap >= 1e-3). Attention: routes come from the oracle on the CPU; P is
rounded to bf16 before the P.V contraction, as in the dense prefill, so outputs are held to
that kernel's bounds: max-abs 1e-2, relative L2 4e-3, lse within 2e-3. Cases cover queries
alone in their block set (groups of one), groups sharing a set with their own biases
(several groups of 128 per set), routes of 32 blocks (two passes of 16), skipped and
zero-probability entries, an empty route and a previous chunk's ring.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import ROUTER_P_ABS, assert_attention_close, to_np

pytestmark = pytest.mark.gpu


def _planted_tokens(plen, cap, T, seed):
    """Per-token router queries: token t uses planted direction t mod 32."""
    pl = synth.plant_router_keys(plen, cap, n_dirs=min(T, 32), seed=seed, device="cuda")
    dirs = torch.arange(T, device="cuda") % pl.q_idx.shape[0]
    q_tok = pl.q_idx[dirs].permute(1, 0, 2).contiguous()              # [B][T][32]
    return pl, q_tok


@pytest.mark.parametrize("plen,cap,T", [([32 * 64, 32 * 40 + 9], 32 * 64, 40), ([32 * 1024] * 2, 32 * 1024, 70),
                                        ([32 * 3200, 8192], 32 * 3200, 33)])
def test_route_tokens_matches_oracle(cuda_lib, plen, cap, T):
    B = len(plen)
    pl, q_tok = _planted_tokens(plen, cap, T, 51)
    pt = torch.tensor(plen, dtype=torch.int32, device="cuda")
    kbar = torch.empty((B, (cap + 31) // 32, 32), dtype=torch.float32, device="cuda")
    cuda_lib.srswa_index_pool(pl.k_idx, pt, kbar)
    blk = torch.empty((B, T, 16), dtype=torch.int32, device="cuda")
    logp = torch.empty((B, T, 16), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    cuda_lib.srswa_route_tokens(q_tok, kbar, pt, blk, logp, ws, prefix_cap=cap)
    assert cuda_lib.check_status(ws) == 0
    o_kbar = oracle.index_pool(to_np(pl.k_idx), np.array(plen, np.int32))
    r_idx, r_logp = oracle.route_tokens(to_np(q_tok), o_kbar, np.array(plen, np.int32))
    np.testing.assert_array_equal(to_np(blk), r_idx)
    np.testing.assert_allclose(np.exp(to_np(logp)), np.exp(r_logp), rtol=0, atol=ROUTER_P_ABS)


def _routes(plen, T, topk, seed):
    rng = np.random.default_rng(seed)
    blk = np.stack([np.stack([rng.permutation((m + 31) // 32)[:topk] for _ in range(T)]) for m in plen])
    logp = np.log(rng.dirichlet(np.ones(topk), size=(len(plen), T)))
    blk[0, 1, min(3, topk - 1)] = -1                                 # a skipped entry
    logp[-1, 2, 0] = -np.inf                                          # a zero-probability entry
    return blk.astype(np.int32), logp.astype(np.float32)


PREFILL_REL_L2 = 4e-3
PREFILL_LSE_ABS = 2e-3


def _check(cuda_lib, d, blk, logp, n, rows, ring=None, tag="", with_lse=True):
    B, H, T, D = d["q"].shape
    out = torch.full((B, H, T, D), float("nan"), dtype=torch.float32, device="cuda")
    lse = torch.full((B, H, T), float("nan"), dtype=torch.float32, device="cuda")
    ws = cuda_lib.srswa_prefill_workspace(B, H, T, d["pk"].shape[2], ring=n)
    kw = {} if ring is None else dict(ring_k=ring["k"], ring_v=ring["v"], wp=ring["wp"], fill=ring["fill"])
    cuda_lib.srswa_prefill(d["q"], d["k_out"], d["v_out"], d["pk"], d["pv"], d["prefix_len"],
                           torch.from_numpy(blk).cuda(), torch.from_numpy(logp).cuda(), out, ws,
                           lse=lse if with_lse else None, scale=d["scale"], ring=n, **kw)
    assert cuda_lib.check_status(ws) == 0
    okw = {} if ring is None else dict(ring_k=to_np(ring["k"]), ring_v=to_np(ring["v"]), wp=to_np(ring["wp"]),
                                       fill=to_np(ring["fill"]))
    ref, ref_lse = oracle.srswa_prefill(to_np(d["q"]), to_np(d["k_out"]), to_np(d["v_out"]), to_np(d["pk"]),
                                        to_np(d["pv"]), to_np(d["prefix_len"]), blk, logp.astype(np.float64),
                                        d["scale"], rows, n, **okw)
    got = to_np(out)[:, :, rows]
    assert_attention_close(got, ref, tag, rel_l2=PREFILL_REL_L2)
    if with_lse:
        assert np.abs(to_np(lse)[:, :, rows] - ref_lse).max() <= PREFILL_LSE_ABS, tag


@pytest.mark.parametrize("plen,cap,T,n", [([1000, 613], 1000, 300, 128), ([200, 33], 200, 90, 40),
                                          ([640, 641], 672, 129, 100)])
def test_srswa_prefill_first_chunk(cuda_lib, plen, cap, T, n):
    d = synth.prefill_case(2, 4, 128, plen, cap, T, seed=61, device="cuda")
    blk, logp = _routes(plen, T, 16 if min(plen) >= 512 else 2, 62)
    _check(cuda_lib, d, blk, logp, n, np.arange(T), tag=f"srswa prefill plen={plen} T={T} n={n}")


@pytest.mark.parametrize("n,wp,fill", [(128, [37, 0], [128, 50]), (40, [3, 39], [40, 7])])
def test_srswa_prefill_with_previous_chunk_ring(cuda_lib, n, wp, fill):
    plen, cap, T = [700, 321], 700, 150
    d = synth.prefill_case(2, 4, 128, plen, cap, T, seed=63, device="cuda")
    c = synth.decode_case(2, 4, 128, 0, 1, n, 1, seed=64, device="cuda", wp0=wp, fill0=fill)
    ring = dict(k=c.ring_k.clone(), v=c.ring_v.clone(), wp=c.wp.clone(), fill=c.fill.clone())
    blk, logp = _routes(plen, T, 8, 65)
    _check(cuda_lib, d, blk, logp, n, np.arange(T), ring=ring, tag=f"srswa prefill ring n={n}")


def test_srswa_prefill_long_history_sampled(cuda_lib):
    # 2 sequences with a 32K-token history, 512 queries per chunk; rows sampled for the oracle
    plen, cap, T = [32768, 30001], 32768, 512
    d = synth.prefill_case(2, 16, 128, plen, cap, T, seed=66, device="cuda", poison=False)
    blk, logp = _routes(plen, T, 16, 67)
    rows = np.concatenate([np.arange(0, 8), np.arange(120, 136), np.arange(T - 8, T)])
    _check(cuda_lib, d, blk, logp, 128, rows, tag="srswa prefill 32K")


def _shared_routes(plen, T, topk, n_sets, seed):
    """Token t routes to block set t mod n_sets (its own entry order and probabilities)."""
    rng = np.random.default_rng(seed)
    B = len(plen)
    blk = np.empty((B, T, topk), np.int32)
    logp = np.empty((B, T, topk), np.float32)
    for b, m in enumerate(plen):
        sets = [rng.permutation((m + 31) // 32)[:topk] for _ in range(n_sets)]
        for t in range(T):
            blk[b, t] = rng.permutation(sets[t % n_sets])
            logp[b, t] = np.log(rng.dirichlet(np.ones(topk)))
    return blk, logp


@pytest.mark.parametrize("plen,cap,T,topk,n_sets", [
    ([1000, 613], 1000, 300, 16, 2),     # 150 queries per set: a group of 128 and one of 22 per set
    ([2048, 1500], 2048, 200, 32, 3),    # 32-block routes: two passes of 16 per group
    ([800, 257], 800, 96, 5, 4),         # short routes (5 blocks: one partial key tile), a partial last block
])
def test_srswa_prefill_shared_block_sets(cuda_lib, plen, cap, T, topk, n_sets):
    d = synth.prefill_case(2, 4, 128, plen, cap, T, seed=71, device="cuda")
    blk, logp = _shared_routes(plen, T, topk, n_sets, 72)
    blk[0, 7, 0] = -1                                      # a skipped entry: that query's set differs
    logp[1, 9, :] = -np.inf                                # an empty route: the band alone
    _check(cuda_lib, d, blk, logp, 128, np.arange(T), tag=f"shared sets plen={plen} T={T} topk={topk}")


def test_srswa_prefill_without_lse(cuda_lib):
    # lse = NULL: the band part's lse lives in the workspace
    plen, cap, T = [700, 321], 700, 150
    d = synth.prefill_case(2, 4, 128, plen, cap, T, seed=73, device="cuda")
    blk, logp = _shared_routes(plen, T, 8, 3, 74)
    _check(cuda_lib, d, blk, logp, 128, np.arange(T), tag="no lse", with_lse=False)


def test_srswa_prefill_bad_block_is_flagged(cuda_lib):
    plen, cap, T = [96, 64], 128, 8
    d = synth.prefill_case(2, 2, 128, plen, cap, T, seed=75, device="cuda")
    blk = np.zeros((2, T, 2), np.int32)
    blk[:, :, 1] = 1
    blk[1, 3, 1] = 3                                       # block 3 of a 64-token (2-block) prefix
    logp = np.full((2, T, 2), np.log(0.5), np.float32)
    out = torch.empty((2, 2, T, 128), dtype=torch.float32, device="cuda")
    ws = cuda_lib.srswa_prefill_workspace(2, 2, T, cap)
    cuda_lib.srswa_prefill(d["q"], d["k_out"], d["v_out"], d["pk"], d["pv"], d["prefix_len"],
                           torch.from_numpy(blk).cuda(), torch.from_numpy(logp).cuda(), out, ws, scale=d["scale"])
    assert cuda_lib.check_status(ws) & cuda_lib.binding.DEVICE_BAD_BLOCK_IDX


def test_srswa_prefill_chunk_full_size_sampled(cuda_lib):
    # the benchmarked chunk: 4 sequences x 16 heads x 4096 queries over a 32K-token history,
    # every query routed by srswa_route_tokens (planted keys, 32 directions cycled over the
    # tokens, so 32 block sets of 128 queries per sequence); routes of sampled tokens against
    # the oracle's router, attention rows sampled against the oracle's prefill
    B, H, T, cap = 4, 16, 4096, 32768
    plen = [cap] * B
    pl = synth.plant_router_keys(plen, cap, n_dirs=32, seed=81, device="cuda")
    q_tok = pl.q_idx[torch.arange(T, device="cuda") % 32].permute(1, 0, 2).contiguous()
    pt = torch.tensor(plen, dtype=torch.int32, device="cuda")
    kbar = torch.empty((B, cap // 32, 32), dtype=torch.float32, device="cuda")
    cuda_lib.srswa_index_pool(pl.k_idx, pt, kbar)
    blk = torch.empty((B, T, 16), dtype=torch.int32, device="cuda")
    logp = torch.empty((B, T, 16), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    cuda_lib.srswa_route_tokens(q_tok, kbar, pt, blk, logp, ws, prefix_cap=cap)
    assert cuda_lib.check_status(ws) == 0
    rows = np.concatenate([np.arange(0, 4), np.arange(126, 131), np.arange(2047, 2050), np.arange(T - 4, T)])
    plen_np = np.array(plen, np.int32)
    r_idx, r_logp = oracle.route_tokens(to_np(q_tok)[:, rows], oracle.index_pool(to_np(pl.k_idx), plen_np), plen_np)
    np.testing.assert_array_equal(to_np(blk)[:, rows], r_idx)
    np.testing.assert_allclose(np.exp(to_np(logp)[:, rows]), np.exp(r_logp), rtol=0, atol=ROUTER_P_ABS)
    del pl
    d = synth.prefill_case(B, H, 128, plen, cap, T, seed=82, device="cuda", poison=False)
    _check(cuda_lib, d, to_np(blk), to_np(logp), 128, rows, tag="srswa prefill full chunk")
