"""Pins the cache-size closed form C(T) = L_m + min(n, T) (and L_m + T for
full attention) against the worked KV-memory example printed in the R-SWA
tutorial page (chenxutan.com/d/4055.html, §5.1), stored in
tests/golden/kv_memory_example.txt."""
import os

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "kv_memory_example.txt")
KB, MB = 1024, 1024 * 1024


def _load():
    vals = {}
    for line in open(GOLDEN, encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        key, val, unit = line.split()
        vals[key] = (float(val), unit)
    return vals


def _bytes(ref, T, layers, window):
    return oracle.kv_cache_bytes(ref, T, heads=32, head_dim=128, layers=layers, bytes_per_elem=2, window=window)


def test_per_token_and_reference():
    g = _load()
    assert _bytes(1, 0, 1, None) == g["per_token_kv"][0] * KB
    assert _bytes(2560, 0, 1, 128) == g["reference_tokens_one_layer"][0] * MB


def test_mha_growth_matches_page():
    g = _load()
    for T in (1024, 4096, 8192, 16384, 32768):
        assert _bytes(2560, T, 1, None) == g[f"mha_one_layer_T{T}"][0] * MB
    # the page's "GB" is 1000 of its MB: 552 MB x 24 = 13248 MB -> 13.2 GB
    assert round(_bytes(2560, 32768, 24, None) / MB / 1000, 1) == g["mha_24_layers_T32768"][0]


def test_rswa_is_constant_and_page_total_is_inconsistent():
    g = _load()
    window_24 = _bytes(0, 32768, 24, 128) / MB
    assert window_24 == 48.0 and abs(window_24 - g["rswa_window_24_layers"][0]) <= 1.2   # page rounds 49152 KB up
    totals = {_bytes(2560, T, 24, 128) for T in (128, 1024, 32768, 10 ** 6)}
    assert totals == {1008 * MB}                      # flat in T once T >= n
    # the printed 90 MB equals the one-layer reference term plus the 24-layer window term
    assert round(_bytes(2560, 0, 1, 128) / MB + g["rswa_window_24_layers"][0]) == \
        g["rswa_total_24_layers_as_printed"][0] - 1
