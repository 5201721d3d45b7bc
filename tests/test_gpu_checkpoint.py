"""Checkpoint / resume of a decode stream.

Everything a decode stream carries from one step to the next is caller-owned: the ring
K/V, wp and fill (the prefix and, for SR-SWA, the block index keys do not change during
decode). Saving those four tensors to host memory mid-run and restoring them into fresh
device buffers, with a fresh workspace, continues the run bit for bit: the kernels are
deterministic (each (sequence, head) output is merged from its split partials in split
order, whichever CTA finishes last). Checked for the fused R-SWA step and for the SR-SWA
step (append + gathered decode): every output, lse, slot and the final state equal an
uninterrupted run's."""
import numpy as np
import pytest
import torch

from long_context_decode_swa_b200 import synth

pytestmark = pytest.mark.gpu

STEPS, CUT = 12, 5


def _fresh_state(case):
    return [case.ring_k.clone(), case.ring_v.clone(), case.wp.clone(), case.fill.clone()]


def _run(rswa, case, state, steps, ws, routes, device):
    ring_k, ring_v, wp, fill = state
    B, H, D = case.q.shape[1:]
    outs = []
    for s in steps:
        out = torch.empty((B, H, D), dtype=torch.float32, device=device)
        lse = torch.empty((B, H), dtype=torch.float32, device=device)
        slot = torch.empty(B, dtype=torch.int32, device=device)
        if routes is None:
            rswa.rswa_decode_append(case.q[s], case.k_new[s], case.v_new[s], case.pk, case.pv, case.prefix_len, ring_k,
                                    ring_v, wp, fill, out, ws, lse=lse, slot_out=slot, scale=case.scale)
        else:
            blk, logp = routes[s]
            rswa.rswa_append(ring_k, ring_v, case.k_new[s], case.v_new[s], wp, fill, slot_out=slot, status=ws)
            rswa.srswa_decode(case.q[s], case.pk, case.pv, case.prefix_len, blk, logp, ring_k, ring_v, wp, fill, out,
                              ws, lse=lse, scale=case.scale)
        outs.append((out, lse, slot))
    return outs


def check_resume(rswa, device, sparse):
    B, H = 4, 8
    plen = [32 * 20, 32 * 33 + 5, 32 * 64, 32 * 17] if sparse else [300, 1000, 77, 2048]
    cap = max(plen)
    case = synth.decode_case(B, H, 128, plen, cap, 128, STEPS, seed=960 + sparse, device=device,
                             wp0=[0, 5, 127, 64], fill0=[0, 128, 50, 127])
    routes = None
    if sparse:
        rng = np.random.default_rng(961)
        routes = []
        for _ in range(STEPS):
            blk = np.stack([rng.permutation((m + 31) // 32)[:16] for m in plen]).astype(np.int32)
            logp = np.log(rng.dirichlet(np.ones(16), B)).astype(np.float32)
            routes.append((torch.from_numpy(blk).to(device), torch.from_numpy(logp).to(device)))
    dims = rswa.dims_of(case.pk, case.ring_k)
    op = rswa.OP_SRSWA_DECODE if sparse else rswa.OP_DECODE

    # the uninterrupted run
    whole_state = _fresh_state(case)
    whole_ws = rswa.new_workspace(dims, op, device)
    whole = _run(rswa, case, whole_state, range(STEPS), whole_ws, routes, device)

    # the same run, checkpointed to host memory after CUT steps and resumed in new buffers
    state = _fresh_state(case)
    ws = rswa.new_workspace(dims, op, device)
    first = _run(rswa, case, state, range(CUT), ws, routes, device)
    saved = [t.to("cpu", copy=True) for t in state]
    assert rswa.check_status(ws) == 0
    del state, ws
    restored = [t.to(device, copy=True) for t in saved]
    ws2 = rswa.new_workspace(dims, op, device)
    rest = _run(rswa, case, restored, range(CUT, STEPS), ws2, routes, device)
    assert rswa.check_status(ws2) == 0 and rswa.check_status(whole_ws) == 0

    for s, (got, want) in enumerate(zip(first + rest, whole)):
        for name, g, w in zip(("out", "lse", "slot"), got, want):
            assert torch.equal(g, w), f"step {s}: {name} differs after resume"
    for name, g, w in zip(("ring_k", "ring_v", "wp", "fill"), restored, whole_state):
        assert torch.equal(g.view(torch.int16) if g.dtype == torch.bfloat16 else g,
                           w.view(torch.int16) if w.dtype == torch.bfloat16 else w), f"final {name} differs"


@pytest.mark.parametrize("sparse", [False, True])
def test_resume_from_a_host_checkpoint_is_bit_exact(cuda_lib, sparse):
    check_resume(cuda_lib, "cuda", sparse)
