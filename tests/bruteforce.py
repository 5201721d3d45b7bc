"""Independent brute-force references used to pin the oracle.

These are written from the pages' definitions in a different form from the
oracle: the R-SWA mask is an explicit [queries x keys] matrix over a flat
token timeline ([R-SWA tutorial] §3.3.1 mask), attention is a dense masked
softmax in torch float64, and the 1.5-entmax threshold is found by bisection
instead of sorting. bf16 widening goes through torch's own bfloat16 dtype.
"""
from __future__ import annotations

import numpy as np
import torch


def u16_to_f64(a: np.ndarray) -> torch.Tensor:
    """bf16 bit patterns (uint16) -> float64 tensor, via torch.bfloat16."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(torch.float64)


def masked_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, visible: torch.Tensor, scale: float,
                     bias: torch.Tensor | None = None):
    """Dense softmax attention with a boolean visibility matrix.

    q [Q][D], k/v [K][D], visible [Q][K] bool, bias [K] or [Q][K] (optional).
    Returns (out [Q][D], lse [Q]).
    """
    Q, D = q.shape
    out = torch.zeros((Q, D), dtype=torch.float64)
    lse = torch.full((Q,), float("-inf"), dtype=torch.float64)
    for r in range(Q):
        idx = torch.nonzero(visible[r]).flatten()
        if idx.numel() == 0:
            continue
        s = scale * (k[idx] @ q[r])
        if bias is not None:
            s = s + (bias[idx] if bias.dim() == 1 else bias[r, idx])
        w = torch.softmax(s, dim=0)
        out[r] = w @ v[idx]
        lse[r] = torch.logsumexp(s, dim=0)
    return out, lse


def rswa_visible(m: int, n: int, query_pos: list[int], n_out: int, first_out: int = 0) -> torch.Tensor:
    """R-SWA visibility over the flat timeline [prefix (m rows); outputs first_out .. first_out+n_out-1].

    Query at output position t sees every prefix row and outputs j with t - n < j <= t.
    """
    K = m + n_out
    vis = torch.zeros((len(query_pos), K), dtype=torch.bool)
    vis[:, :m] = True
    for r, t in enumerate(query_pos):
        for idx in range(n_out):
            j = first_out + idx
            if t - n < j <= t:
                vis[r, m + idx] = True
    return vis


def entmax15_bisect(x: np.ndarray, iters: int = 200):
    """1.5-entmax by bisection on f(tau) = sum max(x - tau, 0)^2 - 1 over [max x - 1, max x]."""
    x = np.asarray(x, np.float64)
    lo, hi = x.max() - 1.0, x.max()
    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        f = np.sum(np.maximum(x - mid, 0.0) ** 2) - 1.0
        if f > 0:
            lo = mid
        else:
            hi = mid
    tau = 0.5 * (lo + hi)
    return np.maximum(x - tau, 0.0) ** 2, tau
