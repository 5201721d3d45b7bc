"""Seeded synthetic inputs for the R-SWA / SR-SWA decode hot path.

This module only draws and lays out inputs; it holds none of the method's
arithmetic (no attention, pooling, scoring, entmax or top-k). Tests, the smoke
check and the benchmark feed the same tensors to the CUDA library and to the
CPU oracle.

Recipe (matches the OCR workloads the pages describe: 256 visual tokens per
page plus a 32-token prompt as the reference prefix, a 128-slot output ring):

* Q, K, V, the ring and the new-token K/V are N(0, 1) drawn in fp32 with a
  seeded ``torch.Generator`` on the target device, then cast to bf16.
* Prefix rows at or past a sequence's prefix length and ring slots that are
  not valid are filled with a NaN poison, so any read of them shows up as NaN.
* SR-SWA router inputs are planted (``plant_router_keys``): for each query
  direction the generator fixes which 16 blocks score highest and in which
  order, with gaps of 0.04 in score, so the top-16 is known by construction.
* An FP8 prefix drawn directly (``fp8_prefix``): uniformly random finite E4M3
  code bytes (the two NaN codes excluded) and log-uniform positive block
  scales, a valid stored cache without going through any quantiser.
* Token positions for the page2d encoding (``page_positions``): consecutive
  output tokens walk through pages of 200-2000 tokens from a random start page
  below 400 and a random offset in it.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BF16_NAN_BITS = 0x7FC0
DI = 32          # router index dimension
BLOCK = 32       # tokens per SR-SWA block
TOPK = 16        # routed blocks per query


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def randn_bf16(shape, gen: torch.Generator, device, std: float = 1.0) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(torch.bfloat16)


def poison_(t: torch.Tensor, mask: torch.Tensor) -> None:
    """Write the bf16 NaN pattern wherever mask (broadcast over trailing dims) is true."""
    t.view(torch.int16)[mask] = BF16_NAN_BITS


def ocr_prefix_len(pages: int, prompt: int = 32, tokens_per_page: int = 256) -> int:
    """Reference prefix length of a document: visual tokens of every page plus the prompt."""
    return pages * tokens_per_page + prompt


@dataclass
class DecodeCase:
    """Inputs of a run of R-SWA / SR-SWA decode steps over B sequences."""
    pk: torch.Tensor           # bf16 [B][H][cap][D]
    pv: torch.Tensor
    prefix_len: torch.Tensor   # int32 [B]
    ring_k: torch.Tensor       # bf16 [B][H][n][D] initial ring contents
    ring_v: torch.Tensor
    wp: torch.Tensor           # int32 [B] initial write pointer
    fill: torch.Tensor         # int32 [B] initial valid-slot count
    q: torch.Tensor            # bf16 [steps][B][H][D]
    k_new: torch.Tensor        # bf16 [steps][B][H][D]
    v_new: torch.Tensor
    scale: float
    extra: dict = field(default_factory=dict)

    @property
    def dims(self):
        B, H, cap, D = self.pk.shape
        return dict(batch=B, heads=H, head_dim=D, ring=self.ring_k.shape[2], prefix_cap=cap)


def decode_case(B: int, H: int, D: int, prefix_len, cap: int, n: int, steps: int, seed: int, device="cpu",
                wp0=None, fill0=None, q_std: float = 1.0, kv_std: float = 1.0, poison: bool = True) -> DecodeCase:
    """Random decode inputs.

    prefix_len: int or sequence of B ints (each <= cap).
    wp0: None (uniform in [0, n)), an int, or a sequence of B ints.
    fill0: None (full ring: n), an int, or a sequence. A ring with fill0 < n has
    its valid slots at (wp0 - fill0 + i) mod n and poison elsewhere.
    """
    g = _gen(seed, device)
    if isinstance(prefix_len, int):
        plen = [prefix_len] * B
    else:
        plen = [int(x) for x in prefix_len]
    assert len(plen) == B and max(plen) <= cap and min(plen) >= 0
    pk = randn_bf16((B, H, cap, D), g, device, kv_std)
    pv = randn_bf16((B, H, cap, D), g, device, kv_std)
    ring_k = randn_bf16((B, H, n, D), g, device, kv_std)
    ring_v = randn_bf16((B, H, n, D), g, device, kv_std)
    if wp0 is None:
        wp = torch.randint(0, n, (B,), generator=g, device=device, dtype=torch.int32)
    elif isinstance(wp0, int):
        wp = torch.full((B,), wp0, dtype=torch.int32, device=device)
    else:
        wp = torch.tensor(list(wp0), dtype=torch.int32, device=device)
    if fill0 is None:
        fill = torch.full((B,), n, dtype=torch.int32, device=device)
    elif isinstance(fill0, int):
        fill = torch.full((B,), fill0, dtype=torch.int32, device=device)
    else:
        fill = torch.tensor(list(fill0), dtype=torch.int32, device=device)
    q = randn_bf16((steps, B, H, D), g, device, q_std)
    k_new = randn_bf16((steps, B, H, D), g, device, kv_std)
    v_new = randn_bf16((steps, B, H, D), g, device, kv_std)
    plen_t = torch.tensor(plen, dtype=torch.int32, device=device)
    if poison:
        rows = torch.arange(cap, device=device)
        bad_rows = rows[None, :] >= plen_t[:, None].to(rows.dtype)           # [B][cap]
        poison_(pk, bad_rows[:, None, :].expand(B, H, cap))
        poison_(pv, bad_rows[:, None, :].expand(B, H, cap))
        slots = torch.arange(n, device=device)
        # slot s is valid iff (s - (wp - fill)) mod n < fill
        age = torch.remainder(slots[None, :] - (wp - fill)[:, None].to(slots.dtype), n)
        bad_slots = age >= fill[:, None].to(slots.dtype)                     # [B][n]
        poison_(ring_k, bad_slots[:, None, :].expand(B, H, n))
        poison_(ring_v, bad_slots[:, None, :].expand(B, H, n))
    return DecodeCase(pk, pv, plen_t, ring_k, ring_v, wp, fill, q, k_new, v_new, 1.0 / math.sqrt(D))


def prefill_case(B: int, H: int, D: int, prefix_len, cap: int, T: int, seed: int, device="cpu",
                 q_std: float = 1.0, poison: bool = True) -> dict:
    """Random chunked-prefill inputs: q/k_out/v_out [B][H][T][D] and a prefix."""
    g = _gen(seed, device)
    plen = [prefix_len] * B if isinstance(prefix_len, int) else [int(x) for x in prefix_len]
    pk = randn_bf16((B, H, cap, D), g, device)
    pv = randn_bf16((B, H, cap, D), g, device)
    q = randn_bf16((B, H, T, D), g, device, q_std)
    k_out = randn_bf16((B, H, T, D), g, device)
    v_out = randn_bf16((B, H, T, D), g, device)
    plen_t = torch.tensor(plen, dtype=torch.int32, device=device)
    if poison:
        rows = torch.arange(cap, device=device)
        bad = (rows[None, :] >= plen_t[:, None].to(rows.dtype))[:, None, :].expand(B, H, cap)
        poison_(pk, bad)
        poison_(pv, bad)
    return dict(q=q, k_out=k_out, v_out=v_out, pk=pk, pv=pv, prefix_len=plen_t, scale=1.0 / math.sqrt(D))


def hadamard32(device="cpu") -> torch.Tensor:
    """Sylvester Hadamard matrix of order 32 (entries +-1, rows mutually orthogonal)."""
    h = torch.ones((1, 1), dtype=torch.float64, device=device)
    while h.shape[0] < DI:
        h = torch.cat([torch.cat([h, h], 1), torch.cat([h, -h], 1)], 0)
    return h


@dataclass
class RouterPlant:
    k_idx: torch.Tensor        # bf16 [B][cap][DI] per-token index keys
    q_idx: torch.Tensor        # fp32 [n_dirs][B][DI] query index vector per direction
    planted: torch.Tensor      # int64 [n_dirs][B][TOPK] planted top blocks, best first
    n_dirs: int


def plant_router_keys(prefix_len, cap: int, n_dirs: int, seed: int, device="cpu", top_hi: float = 4.6,
                      gap: float = 0.04, background: float = 2.0, noise_std: float = 0.5) -> RouterPlant:
    """Index keys with a known top-16 for each of n_dirs query directions.

    Query direction s is row s of a 32x32 Hadamard matrix over sqrt(32), so the
    directions are orthonormal. For each (direction, sequence) the generator
    picks 16 distinct blocks and gives them target scores
    top_hi, top_hi - gap, ..., top_hi - 15 gap; every other block gets a target
    drawn uniformly from [-background, background]. The block centres are the
    combination of the directions weighted by those targets (directions past
    n_dirs carry random weights), so the direction-s query meets centre c at
    exactly its target. Token keys are centre plus antithetic noise (tokens
    2i and 2i+1 of a block get +e and -e), and a partial last block gets
    noise only on complete pairs. Rows past the prefix are NaN poison.
    The defaults give 1.5-entmax supports of exactly the 16 planted blocks
    (targets/2 in [2.0, 2.3], the rest at most 1.0).
    """
    assert 1 <= n_dirs <= DI
    g = _gen(seed, device)
    plen = [int(x) for x in prefix_len]
    B = len(plen)
    nb_cap = (cap + BLOCK - 1) // BLOCK
    Hm = hadamard32(device)                                                   # [DI][DI]
    qs = 1.0 / math.sqrt(DI)
    target = (torch.rand((B, nb_cap, DI), generator=g, device=device, dtype=torch.float64) * 2 - 1) * background
    planted = torch.zeros((n_dirs, B, TOPK), dtype=torch.int64, device=device)
    top_vals = top_hi - gap * torch.arange(TOPK, device=device, dtype=torch.float64)
    for b in range(B):
        nb = (plen[b] + BLOCK - 1) // BLOCK
        assert nb >= TOPK, "planting needs at least 16 blocks"
        for s in range(n_dirs):
            perm = torch.randperm(nb, generator=g, device=device)[:TOPK]
            planted[s, b] = perm
            target[b, perm, s] = top_vals
    # centre_c = (1 / (32 qs)) * sum_s target[c, s] * h_s  so that <qs h_s, centre_c> = target[c, s]
    centre = (target @ Hm) / (DI * qs)                                        # [B][nb_cap][DI]
    noise = torch.randn((B, nb_cap, BLOCK // 2, DI), generator=g, device=device, dtype=torch.float64) * noise_std
    pair = torch.stack([noise, -noise], dim=3).reshape(B, nb_cap, BLOCK, DI)
    keys = centre[:, :, None, :] + pair                                       # [B][nb_cap][BLOCK][DI]
    keys = keys.reshape(B, nb_cap * BLOCK, DI)[:, :cap, :].contiguous()
    for b in range(B):
        m = plen[b]
        tail = m % BLOCK
        if tail:
            c = m // BLOCK
            start = c * BLOCK
            whole = tail - (tail % 2)
            keys[b, start + whole:start + tail, :] = centre[b, c]
    k_idx = keys.to(torch.bfloat16)
    rows = torch.arange(cap, device=device)
    plen_t = torch.tensor(plen, device=device)
    poison_(k_idx, rows[None, :] >= plen_t[:, None])
    q_idx = (Hm[:n_dirs] * qs).to(torch.float32)[:, None, :].expand(n_dirs, B, DI).contiguous()
    return RouterPlant(k_idx, q_idx, planted, n_dirs)


def fp8_prefix(B: int, H: int, cap: int, seed: int, device="cpu", D: int = 128):
    """Random E4M3 codes (uint8 [B][H][cap][D], 0x7f / 0xff excluded) and block scales
    (f32 [B][H][ceil(cap/32)], log-uniform in [2^-10, 2^-4]) for K and for V."""
    g = _gen(seed, device)
    nb = (cap + BLOCK - 1) // BLOCK
    out = []
    for _ in range(2):
        codes = torch.randint(0, 254, (B, H, cap, D), generator=g, device=device, dtype=torch.int32)
        codes = codes + (codes >= 0x7f).int()                          # skip 0x7f; 254 values -> 0..0xfe
        scales = torch.exp2(torch.rand((B, H, nb), generator=g, device=device) * 6.0 - 10.0)
        out += [codes.to(torch.uint8), scales.float()]
    return out[0], out[2], out[1], out[3]                               # k8, v8, k_scale, v_scale


def log_uniform_pages(B: int, lo: int, hi: int, seed: int) -> list[int]:
    """B page counts, log-uniform integers in [lo, hi] (CPU generator, device independent)."""
    g = _gen(seed, "cpu")
    u = torch.rand(B, generator=g, dtype=torch.float64)
    pages = torch.exp(math.log(lo) + u * (math.log(hi + 1) - math.log(lo))).floor().clamp(lo, hi)
    return [int(p) for p in pages]


def page_positions(B: int, T: int, seed: int, page_len=(200, 2000), first_page=(0, 400), device="cpu"):
    """Page layout of T consecutive output tokens per sequence, for the page2d encoding:
    (tok_pos, page), int32 [B][T]. Each sequence starts on a page drawn from
    [first_page[0], first_page[1]) at an offset inside it; pages hold a number of tokens
    drawn from [page_len[0], page_len[1]] (a per-page output length, below the pages'
    20000-token per-page cap); tok_pos is the token's offset inside its page and restarts
    at 0 on each new page. CPU generator, device independent."""
    g = _gen(seed, "cpu")
    lo, hi = page_len
    n_pages = T // lo + 2
    tok = torch.empty((B, T), dtype=torch.int32)
    pg = torch.empty((B, T), dtype=torch.int32)
    for b in range(B):
        lens = torch.randint(lo, hi + 1, (n_pages,), generator=g)
        start_off = int(torch.randint(0, int(lens[0]), (1,), generator=g))
        p0 = int(torch.randint(first_page[0], first_page[1], (1,), generator=g))
        ends = torch.cumsum(lens, 0) - start_off                       # first token index past each page
        t = torch.arange(T)
        j = torch.searchsorted(ends, t, right=True)                   # page (relative) of token t
        begin = torch.where(j > 0, ends[(j - 1).clamp(min=0)], torch.full_like(t, -start_off))
        tok[b] = (t - begin).to(torch.int32)
        pg[b] = (p0 + j).to(torch.int32)
    return tok.to(device), pg.to(device)


def to_u16(t: torch.Tensor):
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    import numpy as np
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
