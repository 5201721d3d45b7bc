"""Page-window scheduling of long documents on top of the decode kernels.

Very long documents are read in windows of pages (ten by default): while a window is
decoded, the reference prefix holds that window's page tokens followed by the prompt;
moving to the next window replaces the prefix and keeps the ring, i.e. the KV tail of
the output generated so far (the Unlimited-OCR serving notes, page-window scheduling:
"the KV tail of the previous window is reused", pages per window configurable, one
window for the whole document when disabled). The prefix length is then bounded by
the window, not by the document: a 400-page book decodes against at most
10 x 256 + 32 prefix tokens.

Host-side bookkeeping only: the prefix and ring live in device tensors that the
library's kernels read; loading a window is a device copy of its page rows.
"""
from __future__ import annotations

import torch

from . import binding as _b


def window_plan(n_pages: int, pages_per_window: int = 10) -> list[range]:
    """The windows of a document: consecutive page ranges of pages_per_window pages (the last may be
    shorter). pages_per_window <= 0 puts the whole document in one window."""
    if n_pages < 0:
        raise ValueError("n_pages must be >= 0")
    if n_pages == 0:
        return []
    w = n_pages if pages_per_window <= 0 else pages_per_window
    return [range(s, min(n_pages, s + w)) for s in range(0, n_pages, w)]


def window_prefix_len(window_pages: int, tokens_per_page: int = 256, prompt_tokens: int = 32) -> int:
    """Prefix tokens while a window of window_pages pages is decoded: its page tokens, then the prompt."""
    return window_pages * tokens_per_page + prompt_tokens


class PageWindowBatch:
    """B documents decoded step by step, each in its current page window.

    Device state: the prefix K/V [B][H][cap][D] (cap = one full window plus the prompt),
    prefix_len [B], and the ring K/V [B][H][n][D] with wp / fill, which starts empty and is
    carried from window to window. Documents advance independently; step() decodes the
    whole batch (append + R-SWA decode)."""

    def __init__(self, pages_per_doc, heads: int = 16, head_dim: int = 128, ring: int = 128,
                 pages_per_window: int = 10, tokens_per_page: int = 256, prompt_tokens: int = 32, device="cuda"):
        self.pages_per_doc = [int(p) for p in pages_per_doc]
        self.B = len(self.pages_per_doc)
        self.H, self.D, self.n = heads, head_dim, ring
        self.tokens_per_page, self.prompt_tokens = tokens_per_page, prompt_tokens
        self.plans = [window_plan(p, pages_per_window) for p in self.pages_per_doc]
        widest = max((len(w) for plan in self.plans for w in plan), default=0)
        self.cap = window_prefix_len(widest, tokens_per_page, prompt_tokens)
        dev = torch.device(device)
        bf16 = dict(dtype=torch.bfloat16, device=dev)
        self.pk = torch.zeros((self.B, heads, self.cap, head_dim), **bf16)
        self.pv = torch.zeros_like(self.pk)
        self.prefix_len = torch.zeros(self.B, dtype=torch.int32, device=dev)
        self.ring_k = torch.zeros((self.B, heads, ring, head_dim), **bf16)
        self.ring_v = torch.zeros_like(self.ring_k)
        self.wp = torch.zeros(self.B, dtype=torch.int32, device=dev)
        self.fill = torch.zeros(self.B, dtype=torch.int32, device=dev)
        self.window = [0 if plan else -1 for plan in self.plans]   # current window per document (-1: none)
        self.workspace = None

    def pages_of(self, b: int) -> range:
        """The pages of document b's current window (empty when the document is finished)."""
        w = self.window[b]
        return self.plans[b][w] if 0 <= w < len(self.plans[b]) else range(0)

    def load_window(self, b: int, page_k: torch.Tensor, page_v: torch.Tensor, prompt_k: torch.Tensor,
                    prompt_v: torch.Tensor) -> int:
        """Write document b's prefix for its current window: page_k / page_v hold the K / V rows of
        exactly the window's pages ([H][pages * tokens_per_page][D] bf16), prompt_k / prompt_v the
        prompt's ([H][prompt_tokens][D]). Returns the new prefix length. The ring is untouched."""
        rows = len(self.pages_of(b)) * self.tokens_per_page
        want = (self.H, rows, self.D)
        if tuple(page_k.shape) != want or tuple(page_v.shape) != want:
            raise ValueError(f"page K/V must be {want} for window {self.window[b]} of document {b}")
        pw = (self.H, self.prompt_tokens, self.D)
        if tuple(prompt_k.shape) != pw or tuple(prompt_v.shape) != pw:
            raise ValueError(f"prompt K/V must be {pw}")
        m = rows + self.prompt_tokens
        self.pk[b, :, :rows].copy_(page_k)
        self.pv[b, :, :rows].copy_(page_v)
        self.pk[b, :, rows:m].copy_(prompt_k)
        self.pv[b, :, rows:m].copy_(prompt_v)
        self.prefix_len[b] = m
        return m

    def advance(self, b: int) -> bool:
        """Move document b to its next window; False when it has none left (its prefix is then
        emptied). The ring, i.e. the KV tail of the previous window's output, is kept."""
        if self.window[b] < 0:
            return False
        self.window[b] += 1
        if self.window[b] >= len(self.plans[b]):
            self.window[b] = -1
            self.prefix_len[b] = 0
            return False
        return True

    def step(self, q, k_new, v_new, out, lse=None, scale=None, stream=None):
        """One decode step of the whole batch: the new tokens join the ring, then every query attends
        to its document's window prefix and ring."""
        if self.workspace is None:
            self.workspace = _b.new_workspace(_b.dims_of(self.pk, self.ring_k), _b.OP_DECODE, self.pk.device)
        _b.rswa_append(self.ring_k, self.ring_v, k_new, v_new, self.wp, self.fill, status=self.workspace,
                       stream=stream)
        _b.rswa_decode(q, self.pk, self.pv, self.prefix_len, self.ring_k, self.ring_v, self.wp, self.fill, out,
                       self.workspace, lse=lse, scale=scale, stream=stream)
