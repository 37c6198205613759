"""Pins for the oracle's cache accounting against the figures the pages print
(tests/golden/page_figures.json, each entry citing its page and section)."""
import json
import os

import pytest

from oracle import mla_oracle as O

G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def test_cached_scalars_per_token():
    g = G["cached_scalars_per_token"]
    assert O.cached_scalars_per_token(g["d_c"], g["d_rope"]) == g["value"]


def test_reduction_vs_32_head_mha():
    r = O.cache_reduction(G["cached_scalars_per_token"]["value"], G["mha32_scalars_per_token"]["value"])
    assert round(100 * r, 2) == G["reduction_vs_mha32_pct"]["value"]


def test_content_compression():
    g = G["content_scalars_mha128"]
    assert g["n_heads"] * g["d_h"] * 2 == g["value"]
    frac = 512 / g["value"]
    assert round(100 * frac, 2) == G["content_compression_pct"]["value"]
    assert round(100 * (1 - frac), 2) == G["content_reduction_pct"]["value"]


def test_h100_speed_of_light_example():
    g = G["h100_example"]
    step = g["batch"] * g["per_stream_gb"]
    assert step == pytest.approx(g["bytes_per_step_gb"], rel=1e-12)
    t = O.transfer_time_s(step * 1e9, g["hbm_gb_per_s"] * 1e9)
    assert round(t * 1e3, 1) == g["ms_per_token"]
    assert round(1 / t, 1) == g["tokens_per_s"]


def test_mha_formula_is_linear_and_factor_two():
    b = G["mha_formula_bytes_per_element"]["bf16"]
    one = O.mha_cache_bytes(1, 1, 1, b, 1, 1)
    assert one == 2 * b
    assert O.mha_cache_bytes(80, 8, 128, b, 8, 1000) == one * 80 * 8 * 128 * 8 * 1000


def test_latent_bytes_per_token():
    n = G["cached_scalars_per_token"]["value"]
    assert O.cache_bytes_per_token(512, 64, "bf16") == n * G["mha_formula_bytes_per_element"]["bf16"]
    assert O.cache_bytes_per_token(512, 64, "f32") == 4 * n
    # fp8: one byte per latent scalar, bf16 k^R, one fp32 scale per 128 latents
    assert O.cache_bytes_per_token(512, 64, "fp8") == 512 + 128 + 16
