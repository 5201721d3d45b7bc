"""GPU parity of the SR-SWA chunked prefill (per-token router + gathered attention over
routed blocks and the causal band) against the oracle.

Routes: block indices bit-exact, probabilities within 1e-5 (planted keys keep every
decisive score gap >= 1e-3). Attention: routes come from the oracle on the CPU; outputs
within max-abs 1e-2 and relative L2 1e-4, lse within 1e-4 (fp32 P, as in decode).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, ROUTER_P_ABS, assert_attention_close, to_np

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


def _check(cuda_lib, d, blk, logp, n, rows, ring=None, tag=""):
    B, H, T, D = d["q"].shape
    out = torch.empty((B, H, T, D), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H, T), dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    kw = {} if ring is None else dict(ring_k=ring["k"], ring_v=ring["v"], wp=ring["wp"], fill=ring["fill"])
    cuda_lib.srswa_prefill(d["q"], d["k_out"], d["v_out"], d["pk"], d["pv"], d["prefix_len"],
                           torch.from_numpy(blk).cuda(), torch.from_numpy(logp).cuda(), out, ws, lse=lse,
                           scale=d["scale"], ring=n, **kw)
    assert cuda_lib.check_status(ws) == 0
    okw = {} if ring is None else dict(ring_k=to_np(ring["k"]), ring_v=to_np(ring["v"]), wp=to_np(ring["wp"]),
                                       fill=to_np(ring["fill"]))
    ref, ref_lse = oracle.srswa_prefill(to_np(d["q"]), to_np(d["k_out"]), to_np(d["v_out"]), to_np(d["pk"]),
                                        to_np(d["pv"]), to_np(d["prefix_len"]), blk, logp.astype(np.float64),
                                        d["scale"], rows, n, **okw)
    got = to_np(out)[:, :, rows]
    assert_attention_close(got, ref, tag)
    assert np.abs(to_np(lse)[:, :, rows] - ref_lse).max() <= LSE_ABS, tag


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
