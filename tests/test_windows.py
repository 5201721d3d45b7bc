"""Page-window scheduling (the Unlimited-OCR serving notes: very long documents are
decoded in windows of pages, ten by default, and the previous window's KV tail is
reused).

CPU: the window plan, the prefix length bound and the batch bookkeeping.
GPU: decoding two documents window by window, with the ring carried across windows,
equals the oracle's decode over each window's prefix and the same ring history.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_swa_b200 import synth, windows
from tests.gpu_util import LSE_ABS, assert_attention_close, to_np


def test_window_plan():
    assert windows.window_plan(25, 10) == [range(0, 10), range(10, 20), range(20, 25)]
    assert windows.window_plan(10, 10) == [range(0, 10)]
    assert windows.window_plan(3, 10) == [range(0, 3)]
    assert windows.window_plan(0, 10) == []
    assert windows.window_plan(25, 0) == [range(0, 25)]          # disabled: one window per document
    pages = [p for w in windows.window_plan(403, 10) for p in w]
    assert pages == list(range(403))                              # every page once, in order


def test_prefix_is_bounded_by_the_window():
    # a 400-page book decodes against at most 10 x 256 + 32 prefix tokens
    plan = windows.window_plan(400, 10)
    assert max(windows.window_prefix_len(len(w)) for w in plan) == 2592
    assert windows.window_prefix_len(len(windows.window_plan(400, 0)[0])) == 400 * 256 + 32


def test_batch_bookkeeping_on_cpu():
    wb = windows.PageWindowBatch([25, 13, 0], heads=2, head_dim=128, ring=16, device="cpu")
    assert wb.cap == 10 * 256 + 32
    assert wb.pages_of(0) == range(0, 10) and wb.pages_of(1) == range(0, 10) and wb.pages_of(2) == range(0)
    z = lambda rows: torch.zeros((2, rows, 128), dtype=torch.bfloat16)
    assert wb.load_window(1, z(2560), z(2560), z(32), z(32)) == 2592
    with pytest.raises(ValueError):
        wb.load_window(0, z(256), z(256), z(32), z(32))          # not the window's page count
    assert wb.advance(1) and wb.pages_of(1) == range(10, 13)
    assert wb.load_window(1, z(768), z(768), z(32), z(32)) == 800
    assert not wb.advance(1) and int(wb.prefix_len[1]) == 0 and wb.pages_of(1) == range(0)
    assert not wb.advance(2)
    assert wb.advance(0) and wb.advance(0) and wb.pages_of(0) == range(20, 25) and not wb.advance(0)


@pytest.mark.gpu
def test_windowed_decode_matches_oracle(cuda_lib):
    pages, H, n, tpp, prompt, steps = [25, 13], 4, 128, 256, 32, 6
    g = torch.Generator(device="cuda").manual_seed(808)
    doc_k = [synth.randn_bf16((H, p * tpp, 128), g, "cuda") for p in pages]
    doc_v = [synth.randn_bf16((H, p * tpp, 128), g, "cuda") for p in pages]
    prompt_k = synth.randn_bf16((2, H, prompt, 128), g, "cuda")
    prompt_v = synth.randn_bf16((2, H, prompt, 128), g, "cuda")
    wb = windows.PageWindowBatch(pages, heads=H, ring=n, tokens_per_page=tpp, prompt_tokens=prompt)
    B = len(pages)
    o_rk = np.zeros((B, H, n, 128), np.uint16)
    o_rv = np.zeros_like(o_rk)
    o_wp = np.zeros(B, np.int32)
    o_fill = np.zeros(B, np.int32)
    out = torch.empty((B, H, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    for w in range(3):                                            # document 1 has 2 windows, document 0 has 3
        # the oracle's prefix is built on the host from the documents' pages, independently of the batch
        o_pk = np.zeros((B, H, wb.cap, 128), np.uint16)
        o_pv = np.zeros_like(o_pk)
        o_plen = np.zeros(B, np.int32)
        for b in range(B):
            plan = windows.window_plan(pages[b], 10)
            if w < len(plan):
                rows = slice(plan[w].start * tpp, plan[w].stop * tpp)
                r = len(plan[w]) * tpp
                o_pk[b, :, :r], o_pv[b, :, :r] = to_np(doc_k[b][:, rows]), to_np(doc_v[b][:, rows])
                o_pk[b, :, r:r + prompt], o_pv[b, :, r:r + prompt] = to_np(prompt_k[b]), to_np(prompt_v[b])
                o_plen[b] = r + prompt
                wb.load_window(b, doc_k[b][:, rows], doc_v[b][:, rows], prompt_k[b], prompt_v[b])
        np.testing.assert_array_equal(to_np(wb.prefix_len), o_plen)
        for s in range(steps):
            q = synth.randn_bf16((B, H, 128), g, "cuda")
            kn = synth.randn_bf16((B, H, 128), g, "cuda")
            vn = synth.randn_bf16((B, H, 128), g, "cuda")
            wb.step(q, kn, vn, out, lse=lse)
            oracle.append(o_rk, o_rv, to_np(kn), to_np(vn), o_wp, o_fill)
            ref, ref_lse = oracle.rswa_decode(to_np(q), o_pk, o_pv, o_plen, o_rk, o_rv, o_wp.copy(), o_fill.copy(),
                                              1.0 / np.sqrt(128))
            assert_attention_close(to_np(out), ref, f"window {w} step {s}")
            assert np.abs(to_np(lse) - ref_lse).max() <= LSE_ABS
        for b in range(B):
            wb.advance(b)
    np.testing.assert_array_equal(to_np(wb.wp), o_wp)          # the ring carried over all windows
    assert int(o_fill[0]) == 18 and wb.window == [-1, -1]
    assert cuda_lib.check_status(wb.workspace) == 0
