"""GPU parity of the SR-SWA path (index pooling, router, gathered-block decode)
against the oracle.

Selected block indices are compared bit-exactly on planted inputs (score gaps
>= 0.04, asserted >= 1e-3 on the oracle's scores); router probabilities and
tau within 1e-5; attention outputs within max-abs 1e-2 and relative L2 1e-4.
On random (unplanted) scores, where near-ties can exist, the unique parts are
compared (probabilities, the multiset of top scores) and the selection is
checked to be a valid top-k.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, ROUTER_P_ABS, DecodeRunner, assert_attention_close, to_np

pytestmark = pytest.mark.gpu


def _route_gpu(rswa, q_idx, kbar, plen_t, cap, topk=16):
    B, nb_cap, _ = kbar.shape
    blk = torch.empty((B, topk), dtype=torch.int32, device="cuda")
    logp = torch.empty((B, topk), dtype=torch.float32, device="cuda")
    probs = torch.empty((B, nb_cap), dtype=torch.float32, device="cuda")
    tau = torch.empty((B,), dtype=torch.float32, device="cuda")
    ws = rswa.route_workspace(B, cap)
    rswa.srswa_route(q_idx, kbar, plen_t, blk, logp, ws, probs=probs, tau=tau, prefix_cap=cap)
    rswa.srswa_route(q_idx, kbar, plen_t, blk, logp, ws, probs=probs, tau=tau, prefix_cap=cap)  # reuse: counters reset
    assert rswa.check_status(ws) == 0
    return to_np(blk), to_np(logp), to_np(probs), to_np(tau)


def test_index_pool_matches_oracle(cuda_lib):
    plen = [32 * 40 + 5, 32 * 16, 32 * 100, 17]
    cap = 32 * 101
    pl = synth.plant_router_keys(plen[:3], cap, n_dirs=2, seed=301, device="cuda")
    k_idx = torch.cat([pl.k_idx, synth.randn_bf16((1, cap, 32), torch.Generator("cuda").manual_seed(3), "cuda")])
    plen_t = torch.tensor(plen, dtype=torch.int32, device="cuda")
    kbar = torch.full((4, (cap + 31) // 32, 32), float("nan"), dtype=torch.float32, device="cuda")
    cuda_lib.srswa_index_pool(k_idx, plen_t, kbar)
    ref = oracle.index_pool(to_np(k_idx), np.array(plen, np.int32))
    got = to_np(kbar)
    np.testing.assert_allclose(got, ref, rtol=0, atol=2e-6)
    assert (got[3, 1:] == 0).all()                  # blocks past a 17-token prefix are zero


@pytest.mark.parametrize("plen", [[32 * 40, 32 * 23 + 5, 32 * 16, 32 * 200], [32 * 1024] * 3, [32 * 3200, 8192]])
def test_route_planted_matches_oracle(cuda_lib, plen):
    cap = max(plen)
    pl = synth.plant_router_keys(plen, cap, n_dirs=6, seed=302, device="cuda")
    plen_t = torch.tensor(plen, dtype=torch.int32, device="cuda")
    nb_cap = (cap + 31) // 32
    kbar = torch.empty((len(plen), nb_cap, 32), dtype=torch.float32, device="cuda")
    cuda_lib.srswa_index_pool(pl.k_idx, plen_t, kbar)
    o_kbar = oracle.index_pool(to_np(pl.k_idx), np.array(plen, np.int32))
    for s in range(pl.n_dirs):
        blk, logp, probs, tau = _route_gpu(cuda_lib, pl.q_idx[s], kbar, plen_t, cap)
        r = oracle.route(to_np(pl.q_idx[s]), o_kbar, np.array(plen, np.int32))
        for b, m in enumerate(plen):
            nb = (m + 31) // 32
            zs = np.sort(r["z"][b, :nb])[::-1]
            assert np.min(zs[:min(16, nb - 1)] - zs[1:min(17, nb)]) >= 1e-3
        np.testing.assert_array_equal(blk, r["blk_idx"])
        np.testing.assert_array_equal(blk, to_np(pl.planted[s]))
        np.testing.assert_allclose(probs, r["probs"], rtol=0, atol=ROUTER_P_ABS)
        np.testing.assert_allclose(tau, r["tau"], rtol=0, atol=ROUTER_P_ABS)
        np.testing.assert_allclose(np.exp(logp), np.exp(r["blk_logp"]), rtol=0, atol=ROUTER_P_ABS)


@pytest.mark.parametrize("seed,nb,spread", [(1, 1000, 1.0), (2, 3000, 0.2), (3, 64, 3.0), (4, 8192, 0.02)])
def test_route_random_scores(cuda_lib, seed, nb, spread):
    # unplanted scores: many entmax candidates (spread 0.02: every block is one); near-ties possible
    rng = np.random.default_rng(seed)
    B = 3
    kbar_np = (rng.normal(0, spread, (B, nb, 32))).astype(np.float32)
    q_np = rng.normal(0, 1, (B, 32)).astype(np.float32)
    plen = [nb * 32, nb * 32 - 31, nb * 16]
    kbar = torch.from_numpy(kbar_np).cuda()
    blk, logp, probs, tau = _route_gpu(cuda_lib, torch.from_numpy(q_np).cuda(), kbar,
                                       torch.tensor(plen, dtype=torch.int32, device="cuda"), nb * 32)
    r = oracle.route(q_np, kbar_np.astype(np.float64), np.array(plen, np.int32))
    np.testing.assert_allclose(probs, r["probs"], rtol=0, atol=ROUTER_P_ABS)
    np.testing.assert_allclose(tau, r["tau"], rtol=0, atol=ROUTER_P_ABS)
    for b in range(B):
        z = r["z"][b]
        assert len(set(blk[b].tolist())) == 16                      # distinct blocks
        np.testing.assert_allclose(np.sort(z[blk[b]])[::-1], np.sort(z[: (plen[b] + 31) // 32])[::-1][:16],
                                   rtol=0, atol=1e-5)                # the 16 largest scores
        assert (np.diff(z[blk[b]]) <= 1e-5).all()                    # in descending order


def test_route_ties_short_and_empty_histories(cuda_lib):
    nb_cap = 20
    kbar = np.zeros((3, nb_cap, 32), np.float32)
    kbar[0, :, 0] = [1, 3, 3, 2, 3, 0, 1, 1, 2, 2, 3, 3, 3, 0, 0, 0, 1, 2, 3, 3]
    kbar[1, :3, 0] = [0.5, 0.25, 0.75]
    q = np.zeros((3, 32), np.float32)
    q[:, 0] = 1.0
    plen = [20 * 32, 3 * 32 - 4, 0]
    blk, logp, probs, tau = _route_gpu(cuda_lib, torch.from_numpy(q).cuda(), torch.from_numpy(kbar).cuda(),
                                       torch.tensor(plen, dtype=torch.int32, device="cuda"), nb_cap * 32, topk=8)
    r = oracle.route(q, kbar.astype(np.float64), np.array(plen, np.int32), topk=8)
    np.testing.assert_array_equal(blk, r["blk_idx"])
    np.testing.assert_array_equal(blk[0], [1, 2, 4, 10, 11, 12, 18, 19])
    np.testing.assert_array_equal(blk[1], [2, 0, 1, -1, -1, -1, -1, -1])
    assert (blk[2] == -1).all() and np.isneginf(logp[2]).all() and (probs[2] == 0).all()
    np.testing.assert_allclose(probs[:2], r["probs"][:2], rtol=0, atol=ROUTER_P_ABS)


def _route_case(plen, cap, n_dirs, seed):
    pl = synth.plant_router_keys(plen, cap, n_dirs=n_dirs, seed=seed, device="cuda")
    o_kbar = oracle.index_pool(to_np(pl.k_idx), np.array(plen, np.int32))
    return pl, o_kbar


def test_srswa_decode_given_route_matches_oracle(cuda_lib):
    # the same route (the oracle's, rounded to fp32) fed to both sides isolates the gathered decode
    plen = [32 * 40 + 9, 32 * 64, 32 * 17]
    cap = 32 * 64
    c = synth.decode_case(3, 16, 128, plen, cap, 128, 4, seed=311, device="cuda", wp0=[5, 0, 127],
                          fill0=[128, 37, 128])
    pl, o_kbar = _route_case(plen, cap, 4, 312)
    r = DecodeRunner(cuda_lib, c)
    for s in range(4):
        ro = oracle.route(to_np(pl.q_idx[s]), o_kbar, np.array(plen, np.int32))
        blk = torch.from_numpy(ro["blk_idx"]).cuda()
        logp32 = ro["blk_logp"].astype(np.float32)
        r.step(s, sparse=(blk, torch.from_numpy(logp32).cuda()))
        ref, ref_lse = r.oracle_srswa(s, ro["blk_idx"], logp32.astype(np.float64))
        got, got_lse = r.gpu_out()
        assert_attention_close(got, ref, f"srswa step {s}")
        assert np.abs(got_lse - ref_lse).max() <= LSE_ABS
    assert cuda_lib.check_status(r.ws_sparse) == 0


def _chain(rswa, plen, cap, B, steps, sample, seed):
    """append -> route -> srswa_decode on the GPU; the oracle runs its own route and decode."""
    c = synth.decode_case(B, 16, 128, plen, cap, 128, steps, seed=seed, device="cuda")
    pl, o_kbar = _route_case(plen, cap, steps, seed + 1)
    plen_t = c.prefix_len
    nb_cap = (cap + 31) // 32
    kbar = torch.empty((B, nb_cap, 32), dtype=torch.float32, device="cuda")
    rswa.srswa_index_pool(pl.k_idx, plen_t, kbar)
    blk = torch.empty((B, 16), dtype=torch.int32, device="cuda")
    logp = torch.empty((B, 16), dtype=torch.float32, device="cuda")
    ws_r = rswa.route_workspace(B, cap)
    r = DecodeRunner(rswa, c, sample)
    for s in range(steps):
        rswa.srswa_route(pl.q_idx[s], kbar, plen_t, blk, logp, ws_r, prefix_cap=cap)
        r.step(s, sparse=(blk, logp))
        ro = oracle.route(to_np(pl.q_idx[s]), o_kbar, np.array(plen, np.int32))
        np.testing.assert_array_equal(to_np(blk), ro["blk_idx"], err_msg=f"step {s}")
        np.testing.assert_allclose(np.exp(to_np(logp)), np.exp(ro["blk_logp"]), rtol=0, atol=ROUTER_P_ABS)
        ref, ref_lse = r.oracle_srswa(s, ro["blk_idx"], ro["blk_logp"])
        got, got_lse = r.gpu_out()
        assert_attention_close(got, ref, f"chain step {s}")
        assert np.abs(got_lse - ref_lse).max() <= LSE_ABS
    r.check_ring()
    assert rswa.check_status(ws_r) == 0 and rswa.check_status(r.ws_sparse) == 0


def test_srswa_chain_32k_history_sampled(cuda_lib):
    # 64 sequences of 32768 tokens (1024 blocks); oracle route for all, oracle decode for 8
    _chain(cuda_lib, [32768] * 64, 32768, 64, 3, np.arange(0, 64, 8), seed=4001)


def test_srswa_chain_ragged_long_horizon(cuda_lib):
    # 16 sequences, 8192..102400 tokens (log-uniform page counts x 256)
    pages = synth.log_uniform_pages(16, 32, 400, seed=5005)
    plen = [256 * p for p in pages]
    sample = sorted({int(np.argmax(plen)), int(np.argmin(plen)), 5, 11})
    _chain(cuda_lib, plen, 102400, 16, 3, np.array(sample), seed=5001)


def test_srswa_all_blocks_zero_bias_equals_rswa(cuda_lib):
    plen = [32 * 20 + 3, 32 * 32]
    cap = 32 * 32
    c = synth.decode_case(2, 16, 128, plen, cap, 128, 1, seed=321, device="cuda")
    r = DecodeRunner(cuda_lib, c)
    blk = torch.tensor([list(range(21)) + [-1] * 11, list(range(31, -1, -1))], dtype=torch.int32, device="cuda")
    logp = torch.zeros((2, 32), dtype=torch.float32, device="cuda")
    logp[0, 21:] = float("-inf")
    r.step(0, sparse=(blk, logp))
    sparse_out = r.out.clone()
    cuda_lib.rswa_decode(c.q[0], c.pk, c.pv, c.prefix_len, r.ring_k, r.ring_v, r.wp, r.fill, r.out, r.ws,
                         scale=c.scale)
    assert_attention_close(to_np(sparse_out), to_np(r.out), "all blocks", rel_l2=1e-6, max_abs=1e-6)


def test_srswa_bad_block_index_is_flagged(cuda_lib):
    c = synth.decode_case(1, 2, 128, 64, 64, 8, 1, seed=331, device="cuda")
    r = DecodeRunner(cuda_lib, c)
    blk = torch.tensor([[0, 2]], dtype=torch.int32, device="cuda")       # block 2 does not exist (2 blocks)
    logp = torch.zeros((1, 2), dtype=torch.float32, device="cuda")
    r.step(0, sparse=(blk, logp))
    assert cuda_lib.check_status(r.ws_sparse) & cuda_lib.binding.DEVICE_BAD_BLOCK_IDX
