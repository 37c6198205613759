"""The C-ABI library without a GPU: it loads, exports every entry point the
header declares, and its host-side checks (dims, page layout, workspace and
argument validation) behave as documented.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

from latent_compressed_attention_mla_b200 import binding as B
from latent_compressed_attention_mla_b200 import workloads as W
from latent_compressed_attention_mla_b200.paged_cache import PagedLatentCache
from oracle import mla_oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_entry_points():
    src = open(os.path.join(ROOT, "include", "mla.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mla_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    L = B.lib()
    names = header_entry_points()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(B.EXPORTED)


@pytest.mark.parametrize("cfg", W.CONFIGS, ids=lambda c: c.name)
def test_page_bytes_match_accounting(cfg):
    d = B.dims_for(cfg)
    assert B.check_dims(d) == 0
    pb = B.cache_page_bytes(d)
    assert pb == PagedLatentCache.layout_page_bytes(d)
    per_token = O.cache_bytes_per_token(cfg.d_c, cfg.d_rope, cfg.cache_dtype)
    assert pb == cfg.page_size * per_token  # no padding for these dims


def test_v3_row_is_576_scalars():
    d = B.dims_for(W.V3_B1_L4096)
    assert B.cache_page_bytes(d) == 64 * 576 * 2


@pytest.mark.parametrize("field,value,code", [
    ("d_c", 24, 1), ("d_rope", 3, 1), ("d_model", 100, 1), ("act_dtype", 7, 1), ("cache_dtype", 9, 1),
    ("softmax_scale", 0.0, 1), ("softmax_scale", float("inf"), 1), ("rope_base", -1.0, 1), ("n_heads", 0, 1)])
def test_invalid_dims_rejected(field, value, code):
    d = B.dims_for(W.V3_B1_L4096)
    setattr(d, field, value)
    assert B.check_dims(d) == code
    assert B.cache_page_bytes(d) == 0


def test_unsupported_combinations():
    d = B.dims_for(W.V3_B1_L4096)
    d.cache_dtype = B.MLA_F32  # fp32 cache needs fp32 activations
    assert B.check_dims(d) == 2
    d = B.dims_for(W.V3_FP8_B128_T2)
    d.d_c = 496  # FP8 tiles are 128 wide
    assert B.check_dims(d) == 2


def test_error_strings():
    for code in range(0, 9):
        assert B.error_string(code)
    assert B.error_string(12345) == "unknown error"


def _p(x):
    return ctypes.c_void_p(x)


def test_host_side_argument_errors_return_before_any_launch():
    L, d = B.lib(), B.dims_for(W.V3_B1_L4096)
    ref = ctypes.byref(d)
    fake = _p(0x10000)  # never dereferenced: validation fails first
    ws_need = B.decode_workspace_bytes(d, 1, 1, 4)
    assert ws_need > 0
    # workspace too small
    assert L.mla_decode(ref, fake, fake, fake, fake, 10, fake, 2, fake, 1, 1, 4, fake, ws_need - 1, None) == 3
    # null query
    assert L.mla_decode(ref, None, fake, fake, fake, 10, fake, 2, fake, 1, 1, 4, fake, ws_need, None) == 1
    # misaligned cache pool
    assert L.mla_decode(ref, fake, fake, fake, _p(0x10008), 10, fake, 2, fake, 1, 1, 4, fake, ws_need, None) == 4
    # bad batch
    assert L.mla_decode(ref, fake, fake, fake, fake, 10, fake, 2, fake, 0, 1, 4, fake, ws_need, None) == 1
    # combine: workspace too small / null output
    assert L.mla_combine(ref, fake, 1, 1, 4, fake, ws_need - 256, fake, None, None) == 3
    assert L.mla_combine(ref, fake, 1, 1, 4, fake, ws_need, None, None, None) == 1
    # append: zero tokens is a no-op, workspace checked otherwise
    assert L.mla_append_latent(ref, None, 0, None, None, None, None, None, 1, 1, None, 1, None, 0, None) == 0
    # bf16/fp32 caches: the projection writes the cache directly, no scratch
    assert B.append_workspace_bytes(d, 3) == 0
    assert L.mla_append_latent(ref, _p(0x10002), 3, fake, fake, fake, fake, fake, 1, 1, fake, 1, None, 0,
                               None) == 4
    # FP8 caches keep fp32 c between the projection and the quantiser
    d8 = B.dims_for(W.V3_FP8_B128_T2)
    ref8 = ctypes.byref(d8)
    need = B.append_workspace_bytes(d8, 3)
    assert need >= 3 * 512 * 4
    assert L.mla_append_latent(ref8, fake, 3, fake, fake, fake, fake, fake, 1, 1, fake, 1, fake, need - 1, None) == 3
    assert L.mla_append_latent(ref8, fake, 3, fake, fake, fake, fake, fake, 1, 1, fake, 1, None, need, None) == 3


def test_workspace_layout_grows_with_splits():
    d = B.dims_for(W.V3_LONG_B8)
    a = B.decode_workspace_bytes(d, 8, 1, 10)
    b = B.decode_workspace_bytes(d, 8, 1, 20)
    # each extra split adds one slot of n_h * (d_c + 1) floats
    assert b - a >= 10 * 128 * 513 * 4 - 512


def test_prefill_workspace_query():
    d = B.dims_for(W.V3_B1_L4096)
    n = B.prefill_workspace_bytes(d, 4096)
    # latent rows and k^R (1152 B per key) plus keys and values of 128 heads (64 KB per key)
    assert n >= 4096 * (1152 + 2 * 128 * 128 * 2)
    assert B.prefill_workspace_bytes(d, 0) == 0
    assert B.prefill_workspace_bytes(B.dims_for(W.TINY_F32), 256) == 0  # fp32 / other dims: no prefill kernel


def test_fast_append_workspace_holds_the_split_k_partials():
    """Steps of 16 to 511 tokens (V3 dims, bf16 activations) have a faster
    path whose fp32 partial tiles need more scratch: splits x 128-token tiles
    x 576 outputs, with 3 x tiles x splits CTA tiles at most 144 and at most
    16 splits.  Outside that range the fast size is the minimum."""
    for cfg in (W.V3_B1_L4096, W.V3_FP8_B128_T2):
        d = B.dims_for(cfg)
        for n in (1, 4, 15, 512, 4096):
            assert B.append_workspace_bytes_fast(d, n) == B.append_workspace_bytes(d, n)
        for n in (16, 64, 128, 129, 256, 511):
            m_tiles = -(-n // 128)
            splits = min(144 // (3 * m_tiles), 16, d.d_model // 64)
            fast = B.append_workspace_bytes_fast(d, n)
            assert fast >= splits * m_tiles * 128 * 576 * 4
            assert fast >= B.append_workspace_bytes(d, n)
            assert 3 * m_tiles * splits <= 144
