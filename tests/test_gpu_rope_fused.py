"""GPU parity of the fused decode steps that take the page2d encoding inside the launch
(rswa_decode_append_rope, srswa_step_rope), over several steps in a row whose tokens cross
page boundaries.

Two references on the same seeded inputs:
* the library's unfused sequence: rswa_rope_page2d on q and k_new, then rswa_decode_append
  (resp. srswa_step) on the encoded rows. The fused step takes the same fp64 angles, the
  same f32 cos / sin, the same f32 rotation and the same attention order, so it must give
  the same bits: out, lse, ring bytes, wp, fill, slot_out and, for SR-SWA, the route;
* the oracle: its fp64 encoding rounded to bf16, its append and its decode: outputs within
  max-abs 1e-2 / relative L2 1e-4, lse within 1e-4, and the appended key within the
  encoding bound of the stand-alone kernels (test_gpu_rope.assert_rope_close).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth
from tests.gpu_util import LSE_ABS, ROUTER_P_ABS, assert_attention_close, to_np
from tests.test_gpu_rope import assert_rope_close

pytestmark = pytest.mark.gpu


class Arm:
    """One copy of the ring state and the outputs of a run."""

    def __init__(self, rswa, c, op):
        B, H, cap, D = c.pk.shape
        self.ring_k, self.ring_v = c.ring_k.clone(), c.ring_v.clone()
        self.wp, self.fill = c.wp.clone(), c.fill.clone()
        self.ws = rswa.new_workspace(rswa.dims_of(c.pk, c.ring_k), op)
        self.out = torch.full((B, H, D), float("nan"), dtype=torch.float32, device="cuda")
        self.lse = torch.full((B, H), float("nan"), dtype=torch.float32, device="cuda")
        self.slot = torch.full((B,), -9, dtype=torch.int32, device="cuda")
        self.blk = torch.full((B, 16), -7, dtype=torch.int32, device="cuda")
        self.logp = torch.zeros((B, 16), dtype=torch.float32, device="cuda")
        self.tau = torch.zeros((B,), dtype=torch.float32, device="cuda")

    def assert_same(self, other, what, route=False):
        pairs = [("out", self.out, other.out), ("lse", self.lse, other.lse), ("ring_k", self.ring_k, other.ring_k),
                 ("ring_v", self.ring_v, other.ring_v), ("wp", self.wp, other.wp), ("fill", self.fill, other.fill),
                 ("slot_out", self.slot, other.slot)]
        if route:
            pairs += [("blk_idx", self.blk, other.blk), ("blk_logp", self.logp, other.logp),
                      ("tau", self.tau, other.tau)]
        bits = {torch.float32: torch.int32, torch.bfloat16: torch.int16}  # NaN poison compares by its bits
        for name, a, b in pairs:
            assert torch.equal(a.view(bits.get(a.dtype, a.dtype)), b.view(bits.get(b.dtype, b.dtype))), \
                f"{what}: {name} differs"


class OracleRing:
    """The oracle's ring state, appended with the oracle's encoded keys."""

    def __init__(self, c):
        self.rk, self.rv = to_np(c.ring_k).copy(), to_np(c.ring_v).copy()
        self.wp, self.fill = to_np(c.wp).copy(), to_np(c.fill).copy()

    def append(self, ko, v):
        return oracle.append(self.rk, self.rv, ko, v, self.wp, self.fill)


def _encode(rswa, q, k, tok, page, base, page_mod):
    q_rot, k_rot = torch.empty_like(q), torch.empty_like(k)
    rswa.rswa_rope_page2d(q, tok, page, q_out=q_rot, k=k, k_out=k_rot, base=base, page_mod=page_mod)
    return q_rot, k_rot


@pytest.mark.parametrize("B,H,plen,cap,n,wp0,fill0,steps,base,page_mod", [
    (3, 4, [5, 77, 200], 200, 40, [0, 13, 39], [0, 40, 17], 6, 10000.0, 2),   # empty / full / partial rings
    (2, 8, [9000, 4097], 9000, 128, [5, 127], 128, 3, 10000.0, 2),            # several splits per (b, h)
    (4, 20, [300, 1, 64, 129], 300, 100, None, 100, 4, 500000.0, 3),          # 20 heads, n = 100, page_mod 3
    (2, 16, [288, 288], 288, 128, 37, 128, 3, 10000.0, 0),                    # token axis only
])
def test_decode_append_rope_matches_unfused_and_oracle(cuda_lib, B, H, plen, cap, n, wp0, fill0, steps, base,
                                                       page_mod):
    rswa = cuda_lib
    c = synth.decode_case(B, H, 128, plen, cap, n, steps, seed=950 + H, device="cuda", wp0=wp0, fill0=fill0)
    tok, page = synth.page_positions(B, steps, seed=951 + H, page_len=(2, 4))
    fused, ref = Arm(rswa, c, rswa.OP_DECODE), Arm(rswa, c, rswa.OP_DECODE)
    o = OracleRing(c)
    for s in range(steps):
        t_s, p_s = tok[:, s].contiguous().cuda(), page[:, s].contiguous().cuda()
        rswa.rswa_decode_append_rope(c.q[s], c.k_new[s], c.v_new[s], c.pk, c.pv, c.prefix_len, fused.ring_k,
                                     fused.ring_v, fused.wp, fused.fill, t_s, p_s, fused.out, fused.ws, lse=fused.lse,
                                     slot_out=fused.slot, base=base, page_mod=page_mod, scale=c.scale)
        q_rot, k_rot = _encode(rswa, c.q[s], c.k_new[s], t_s, p_s, base, page_mod)
        rswa.rswa_decode_append(q_rot, k_rot, c.v_new[s], c.pk, c.pv, c.prefix_len, ref.ring_k, ref.ring_v, ref.wp,
                                ref.fill, ref.out, ref.ws, lse=ref.lse, slot_out=ref.slot, scale=c.scale)
        fused.assert_same(ref, f"step {s}")
        # the oracle: encoded rows correctly rounded to bf16, then its append and decode
        ts, ps = tok[:, s].numpy(), page[:, s].numpy()
        qo = oracle.bf16_round(oracle.rope_page2d(to_np(c.q[s]), ts, ps, base=base, page_mod=page_mod))
        ko = oracle.bf16_round(oracle.rope_page2d(to_np(c.k_new[s]), ts, ps, base=base, page_mod=page_mod))
        slot = o.append(ko, to_np(c.v_new[s]))
        np.testing.assert_array_equal(to_np(fused.slot), slot, err_msg=f"slot_out step {s}")
        np.testing.assert_array_equal(to_np(fused.wp), o.wp, err_msg=f"wp step {s}")
        got_rk = to_np(fused.ring_k)
        for b in range(B):
            assert_rope_close(got_rk[b, :, slot[b]][None], to_np(c.k_new[s])[b][None], ts[b:b + 1], ps[b:b + 1],
                              base, page_mod, f"appended key b={b} step {s}")
        np.testing.assert_array_equal(to_np(fused.ring_v), o.rv, err_msg=f"ring_v step {s}")
        want, want_lse = oracle.rswa_decode(qo, to_np(c.pk), to_np(c.pv), to_np(c.prefix_len), o.rk, o.rv, o.wp,
                                            o.fill, c.scale)
        assert_attention_close(to_np(fused.out), want, f"encoded fused step {s}")
        assert np.abs(to_np(fused.lse) - want_lse).max() <= LSE_ABS
    assert rswa.check_status(fused.ws) == 0 and rswa.check_status(ref.ws) == 0


def test_decode_append_rope_bad_ring_state(cuda_lib):
    # a sequence with an out-of-range write pointer: flagged, not appended, its query still encoded;
    # the fused step and the unfused sequence agree bit for bit
    rswa = cuda_lib
    c = synth.decode_case(3, 4, 128, [100, 64, 33], 100, 32, 1, seed=960, device="cuda", wp0=[3, 40, 0],
                          fill0=[32, 10, 0])
    tok, page = synth.page_positions(3, 1, seed=961)
    t_s, p_s = tok[:, 0].contiguous().cuda(), page[:, 0].contiguous().cuda()
    fused, ref = Arm(rswa, c, rswa.OP_DECODE), Arm(rswa, c, rswa.OP_DECODE)
    rswa.rswa_decode_append_rope(c.q[0], c.k_new[0], c.v_new[0], c.pk, c.pv, c.prefix_len, fused.ring_k,
                                 fused.ring_v, fused.wp, fused.fill, t_s, p_s, fused.out, fused.ws, lse=fused.lse,
                                 slot_out=fused.slot, scale=c.scale)
    q_rot, k_rot = _encode(rswa, c.q[0], c.k_new[0], t_s, p_s, 10000.0, 2)
    rswa.rswa_decode_append(q_rot, k_rot, c.v_new[0], c.pk, c.pv, c.prefix_len, ref.ring_k, ref.ring_v, ref.wp,
                            ref.fill, ref.out, ref.ws, lse=ref.lse, slot_out=ref.slot, scale=c.scale)
    assert rswa.check_status(fused.ws) == rswa.binding.DEVICE_BAD_RING_STATE
    assert rswa.check_status(ref.ws) == rswa.binding.DEVICE_BAD_RING_STATE
    fused.assert_same(ref, "bad ring state")
    assert int(fused.slot[1]) == -9 and int(fused.wp[1]) == 40      # untouched


def test_decode_append_rope_batched_workload(cuda_lib):
    # the batched R-SWA decode workload (512 sequences, 10-page prefix, full ring) in the launch
    # configuration the benchmark times: every output bit-equal to the unfused sequence, sampled
    # sequences against the oracle
    rswa = cuda_lib
    m = synth.ocr_prefix_len(10)
    c = synth.decode_case(512, 16, 128, m, m, 128, 2, seed=970, device="cuda")
    tok, page = synth.page_positions(512, 2, seed=971)
    fused, ref = Arm(rswa, c, rswa.OP_DECODE), Arm(rswa, c, rswa.OP_DECODE)
    sample = np.sort(np.random.default_rng(972).choice(512, 8, replace=False))
    o_rk, o_rv = to_np(c.ring_k)[sample].copy(), to_np(c.ring_v)[sample].copy()
    o_wp, o_fill = to_np(c.wp)[sample].copy(), to_np(c.fill)[sample].copy()
    sel = torch.as_tensor(sample, device="cuda")
    o_pk, o_pv = to_np(c.pk.index_select(0, sel)), to_np(c.pv.index_select(0, sel))
    for s in range(2):
        t_s, p_s = tok[:, s].contiguous().cuda(), page[:, s].contiguous().cuda()
        rswa.rswa_decode_append_rope(c.q[s], c.k_new[s], c.v_new[s], c.pk, c.pv, c.prefix_len, fused.ring_k,
                                     fused.ring_v, fused.wp, fused.fill, t_s, p_s, fused.out, fused.ws, lse=fused.lse,
                                     slot_out=fused.slot, scale=c.scale)
        q_rot, k_rot = _encode(rswa, c.q[s], c.k_new[s], t_s, p_s, 10000.0, 2)
        rswa.rswa_decode_append(q_rot, k_rot, c.v_new[s], c.pk, c.pv, c.prefix_len, ref.ring_k, ref.ring_v, ref.wp,
                                ref.fill, ref.out, ref.ws, lse=ref.lse, slot_out=ref.slot, scale=c.scale)
        fused.assert_same(ref, f"batched step {s}")
        ts, ps = tok[sample, s].numpy(), page[sample, s].numpy()
        qo = oracle.bf16_round(oracle.rope_page2d(to_np(c.q[s])[sample], ts, ps))
        ko = oracle.bf16_round(oracle.rope_page2d(to_np(c.k_new[s])[sample], ts, ps))
        oracle.append(o_rk, o_rv, ko, to_np(c.v_new[s])[sample], o_wp, o_fill)
        want, want_lse = oracle.rswa_decode(qo, o_pk, o_pv, to_np(c.prefix_len)[sample], o_rk, o_rv, o_wp, o_fill,
                                            c.scale)
        assert_attention_close(to_np(fused.out)[sample], want, f"batched encoded step {s}")
        assert np.abs(to_np(fused.lse)[sample] - want_lse).max() <= LSE_ABS
    assert rswa.check_status(fused.ws) == 0


@pytest.mark.parametrize("plen,H,steps", [
    ([32 * 40, 32 * 23 + 5, 32 * 16], 4, 4),      # ragged histories, partial last block
    ([32 * 1024] * 2, 16, 3),                     # 32K histories, the SR-SWA decode workload's shape
])
def test_srswa_step_rope_matches_unfused_and_oracle(cuda_lib, plen, H, steps):
    rswa = cuda_lib
    B, cap = len(plen), max(plen)
    c = synth.decode_case(B, H, 128, plen, cap, 128, steps, seed=980 + H, device="cuda", fill0=[128, 60, 0][:B])
    pl = synth.plant_router_keys(plen, cap, n_dirs=4, seed=981 + H, device="cuda")
    plen_t = torch.tensor(plen, dtype=torch.int32, device="cuda")
    kbar = torch.empty((B, (cap + 31) // 32, 32), dtype=torch.float32, device="cuda")
    rswa.srswa_index_pool(pl.k_idx, plen_t, kbar)
    o_kbar = oracle.index_pool(to_np(pl.k_idx), np.array(plen, np.int32))
    tok, page = synth.page_positions(B, steps, seed=982 + H, page_len=(2, 3))
    fused, ref = Arm(rswa, c, rswa.OP_SRSWA_ROUTED), Arm(rswa, c, rswa.OP_SRSWA_ROUTED)
    o = OracleRing(c)
    for s in range(steps):
        t_s, p_s = tok[:, s].contiguous().cuda(), page[:, s].contiguous().cuda()
        rswa.srswa_step_rope(c.q[s], c.k_new[s], c.v_new[s], pl.q_idx[s], kbar, c.pk, c.pv, c.prefix_len,
                             fused.ring_k, fused.ring_v, fused.wp, fused.fill, t_s, p_s, fused.blk, fused.logp,
                             fused.out, fused.ws, lse=fused.lse, tau=fused.tau, slot_out=fused.slot, scale=c.scale)
        q_rot, k_rot = _encode(rswa, c.q[s], c.k_new[s], t_s, p_s, 10000.0, 2)
        rswa.srswa_step(q_rot, k_rot, c.v_new[s], pl.q_idx[s], kbar, c.pk, c.pv, c.prefix_len, ref.ring_k,
                        ref.ring_v, ref.wp, ref.fill, ref.blk, ref.logp, ref.out, ref.ws, lse=ref.lse, tau=ref.tau,
                        slot_out=ref.slot, scale=c.scale)
        fused.assert_same(ref, f"SR-SWA step {s}", route=True)
        # the oracle: the route (the router query is not encoded), the encoded append, the decode
        ro = oracle.route(to_np(pl.q_idx[s]), o_kbar, np.array(plen, np.int32))
        np.testing.assert_array_equal(to_np(fused.blk), ro["blk_idx"], err_msg=f"route step {s}")
        np.testing.assert_allclose(np.exp(to_np(fused.logp)), np.exp(ro["blk_logp"]), rtol=0, atol=ROUTER_P_ABS)
        ts, ps = tok[:, s].numpy(), page[:, s].numpy()
        qo = oracle.bf16_round(oracle.rope_page2d(to_np(c.q[s]), ts, ps))
        ko = oracle.bf16_round(oracle.rope_page2d(to_np(c.k_new[s]), ts, ps))
        slot = o.append(ko, to_np(c.v_new[s]))
        np.testing.assert_array_equal(to_np(fused.slot), slot, err_msg=f"slot_out step {s}")
        want, want_lse = oracle.srswa_decode(qo, to_np(c.pk), to_np(c.pv), np.array(plen, np.int32), ro["blk_idx"],
                                             ro["blk_logp"], o.rk, o.rv, o.wp, o.fill, c.scale)
        assert_attention_close(to_np(fused.out), want, f"encoded SR-SWA step {s}")
        assert np.abs(to_np(fused.lse) - want_lse).max() <= LSE_ABS
    assert rswa.check_status(fused.ws) == 0 and rswa.check_status(ref.ws) == 0


def test_srswa_step_rope_full_size_sampled(cuda_lib):
    # the benchmarked encoded SR-SWA step: 64 sequences x 16 heads, 32K-token histories, two
    # steps; every output bit-equal to the unfused sequence, the route of every sequence against
    # the oracle's router, sampled sequences against the oracle's encoding, append and decode
    rswa = cuda_lib
    B, H, cap, steps = 64, 16, 32768, 2
    plen = [cap] * B
    c = synth.decode_case(B, H, 128, plen, cap, 128, steps, seed=990, device="cuda")
    pl = synth.plant_router_keys(plen, cap, n_dirs=4, seed=991, device="cuda")
    pt = torch.tensor(plen, dtype=torch.int32, device="cuda")
    kbar = torch.empty((B, cap // 32, 32), dtype=torch.float32, device="cuda")
    rswa.srswa_index_pool(pl.k_idx, pt, kbar)
    o_kbar = oracle.index_pool(to_np(pl.k_idx), np.array(plen, np.int32))
    tok, page = synth.page_positions(B, steps, seed=992)
    fused, ref = Arm(rswa, c, rswa.OP_SRSWA_ROUTED), Arm(rswa, c, rswa.OP_SRSWA_ROUTED)
    sample = np.array([0, 9, 31, 63])
    sel = torch.as_tensor(sample, device="cuda")
    o_pk, o_pv = to_np(c.pk.index_select(0, sel)), to_np(c.pv.index_select(0, sel))
    o_rk, o_rv = to_np(c.ring_k)[sample].copy(), to_np(c.ring_v)[sample].copy()
    o_wp, o_fill = to_np(c.wp)[sample].copy(), to_np(c.fill)[sample].copy()
    for s in range(steps):
        t_s, p_s = tok[:, s].contiguous().cuda(), page[:, s].contiguous().cuda()
        rswa.srswa_step_rope(c.q[s], c.k_new[s], c.v_new[s], pl.q_idx[s], kbar, c.pk, c.pv, c.prefix_len,
                             fused.ring_k, fused.ring_v, fused.wp, fused.fill, t_s, p_s, fused.blk, fused.logp,
                             fused.out, fused.ws, lse=fused.lse, tau=fused.tau, slot_out=fused.slot, scale=c.scale)
        q_rot, k_rot = _encode(rswa, c.q[s], c.k_new[s], t_s, p_s, 10000.0, 2)
        rswa.srswa_step(q_rot, k_rot, c.v_new[s], pl.q_idx[s], kbar, c.pk, c.pv, c.prefix_len, ref.ring_k,
                        ref.ring_v, ref.wp, ref.fill, ref.blk, ref.logp, ref.out, ref.ws, lse=ref.lse, tau=ref.tau,
                        slot_out=ref.slot, scale=c.scale)
        fused.assert_same(ref, f"full-size SR-SWA step {s}", route=True)
        ro = oracle.route(to_np(pl.q_idx[s]), o_kbar, np.array(plen, np.int32))
        np.testing.assert_array_equal(to_np(fused.blk), ro["blk_idx"], err_msg=f"route step {s}")
        ts, ps = tok[sample, s].numpy(), page[sample, s].numpy()
        qo = oracle.bf16_round(oracle.rope_page2d(to_np(c.q[s])[sample], ts, ps))
        ko = oracle.bf16_round(oracle.rope_page2d(to_np(c.k_new[s])[sample], ts, ps))
        oracle.append(o_rk, o_rv, ko, to_np(c.v_new[s])[sample], o_wp, o_fill)
        want, want_lse = oracle.srswa_decode(qo, o_pk, o_pv, np.array(plen, np.int32)[sample],
                                             np.ascontiguousarray(ro["blk_idx"][sample]),
                                             np.ascontiguousarray(ro["blk_logp"][sample]), o_rk, o_rv, o_wp, o_fill,
                                             c.scale)
        assert_attention_close(to_np(fused.out)[sample], want, f"full-size encoded SR-SWA step {s}")
        assert np.abs(to_np(fused.lse)[sample] - want_lse).max() <= LSE_ABS
    assert rswa.check_status(fused.ws) == 0 and rswa.check_status(ref.ws) == 0
