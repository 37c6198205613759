"""ctypes binding of libmla (include/mla.h).

Argument marshalling only: every step of the decode path runs in the CUDA
kernels of libmla.so.  torch tensors supply device memory and the current CUDA
stream.  If the library is missing, loading raises; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla.so")

MLA_F32, MLA_BF16, MLA_FP8_E4M3 = 0, 1, 2
MLA_FLAG_FORCE_SIMT = 1
MLA_FLAG_SELFTEST_STALL = 2  # decode issues no loads, combine no weight fetch: bounded waits expire (tests)

(MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_WORKSPACE, MLA_ERR_ALIGNMENT, MLA_ERR_LAUNCH,
 MLA_ERR_TIMEOUT, MLA_ERR_BOUNDS, MLA_ERR_CUDA) = range(9)
ERRORS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
          4: "MLA_ERR_ALIGNMENT", 5: "MLA_ERR_LAUNCH", 6: "MLA_ERR_TIMEOUT", 7: "MLA_ERR_BOUNDS",
          8: "MLA_ERR_CUDA"}

# Every entry point declared in include/mla.h.
EXPORTED = ("mla_cache_page_bytes", "mla_check_dims", "mla_append_workspace_bytes",
            "mla_append_workspace_bytes_fast", "mla_append_latent",
            "mla_append_latent_noalloc",
            "mla_decode_workspace_bytes", "mla_decode", "mla_combine", "mla_prefill_workspace_bytes",
            "mla_prefill", "mla_decode_path", "mla_auto_splits",
            "mla_set_trace_events", "mla_set_timeline", "mla_get_status", "mla_error_string")
TRACE_KERNELS = ("append_project", "append_finalize", "absorb", "attend", "combine",
                 "prefill_prep", "prefill_upproj", "prefill_attend")


class MlaDims(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("d_nope", ctypes.c_int32), ("d_v", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("act_dtype", ctypes.c_int32), ("cache_dtype", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("rope_base", ctypes.c_float), ("flags", ctypes.c_uint32)]


class MlaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {ERRORS.get(code, code)} ({error_string(code)})")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmla.so not built at {LIB_PATH}; run latent_compressed_attention_mla_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.POINTER(MlaDims)
        L.mla_cache_page_bytes.argtypes, L.mla_cache_page_bytes.restype = [S], Z
        L.mla_check_dims.argtypes, L.mla_check_dims.restype = [S], I
        L.mla_append_workspace_bytes.argtypes, L.mla_append_workspace_bytes.restype = [S, I], Z
        L.mla_append_workspace_bytes_fast.argtypes, L.mla_append_workspace_bytes_fast.restype = [S, I], Z
        L.mla_append_latent.argtypes = [S, P, I, P, P, P, P, P, I, I, P, I, P, Z, P]
        L.mla_append_latent.restype = I
        L.mla_append_latent_noalloc.argtypes = [S, P, I, P, P, P, P, P, I, I, P, I, P]
        L.mla_append_latent_noalloc.restype = I
        L.mla_decode_workspace_bytes.argtypes, L.mla_decode_workspace_bytes.restype = [S, I, I, I], Z
        L.mla_decode.argtypes = [S, P, P, P, P, I, P, I, P, I, I, I, P, Z, P]
        L.mla_decode.restype = I
        L.mla_combine.argtypes = [S, P, I, I, I, P, Z, P, P, P]
        L.mla_combine.restype = I
        L.mla_prefill_workspace_bytes.argtypes, L.mla_prefill_workspace_bytes.restype = [S, I], Z
        L.mla_prefill.argtypes = [S, P, P, P, P, P, I, P, I, P, I, I, I, P, Z, P, P, P]
        L.mla_prefill.restype = I
        L.mla_decode_path.argtypes, L.mla_decode_path.restype = [S, I], I
        L.mla_auto_splits.argtypes, L.mla_auto_splits.restype = [S, I, I], I
        L.mla_get_status.argtypes, L.mla_get_status.restype = [P, ctypes.POINTER(ctypes.c_int)], I
        L.mla_error_string.argtypes, L.mla_error_string.restype = [I], ctypes.c_char_p
        L.mla_set_trace_events.argtypes, L.mla_set_trace_events.restype = [ctypes.POINTER(P), I], I
        L.mla_set_timeline.argtypes, L.mla_set_timeline.restype = [P], I
        _lib = L
    return _lib


def error_string(code: int) -> str:
    return lib().mla_error_string(code).decode()


def make_dims(n_heads, d_c, d_rope, d_nope, d_v, d_model, page_size=64, act="bf16", cache="bf16",
              softmax_scale=None, rope_base=10000.0, flags=0) -> MlaDims:
    codes = {"f32": MLA_F32, "bf16": MLA_BF16, "fp8": MLA_FP8_E4M3}
    if softmax_scale is None:
        softmax_scale = (d_nope + d_rope) ** -0.5
    return MlaDims(n_heads, d_c, d_rope, d_nope, d_v, d_model, page_size, codes[act], codes[cache],
                   softmax_scale, rope_base, flags)


def dims_for(cfg, flags: int = 0) -> MlaDims:
    """Dims of a workloads.MlaConfig."""
    return make_dims(cfg.n_heads, cfg.d_c, cfg.d_rope, cfg.d_nope, cfg.d_v, cfg.d_model, cfg.page_size,
                     cfg.act_dtype, cfg.cache_dtype, cfg.softmax_scale, cfg.rope_base, flags)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(rc: int, what: str):
    if rc != 0:
        raise MlaError(rc, what)


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors passed to libmla must be contiguous CUDA tensors")


def cache_page_bytes(dims: MlaDims) -> int:
    return int(lib().mla_cache_page_bytes(ctypes.byref(dims)))


def check_dims(dims: MlaDims) -> int:
    return int(lib().mla_check_dims(ctypes.byref(dims)))


def append_workspace_bytes(dims: MlaDims, n_tokens: int) -> int:
    return int(lib().mla_append_workspace_bytes(ctypes.byref(dims), n_tokens))


def append_workspace_bytes_fast(dims: MlaDims, n_tokens: int) -> int:
    return int(lib().mla_append_workspace_bytes_fast(ctypes.byref(dims), n_tokens))


def decode_workspace_bytes(dims: MlaDims, batch: int, n_q: int, num_splits: int = 0) -> int:
    return int(lib().mla_decode_workspace_bytes(ctypes.byref(dims), batch, n_q, num_splits))


def decode_path(dims: MlaDims, n_q: int) -> int:
    return int(lib().mla_decode_path(ctypes.byref(dims), n_q))


def auto_splits(dims: MlaDims, batch: int, n_q: int) -> int:
    return int(lib().mla_auto_splits(ctypes.byref(dims), batch, n_q))


def mla_append_latent(dims, h, seq_idx, pos, W_dkv, W_kr, page_table, cache_pool, workspace, stream=None):
    """S1: append the rows of h [N, d_model] at (seq_idx[n], pos[n]).  page_table
    [batch, max_pages] int32; cache_pool a uint8 tensor of num_pages pages."""
    _cuda(h, seq_idx, pos, W_dkv, W_kr, page_table, cache_pool, workspace)
    num_pages = cache_pool.numel() * cache_pool.element_size() // cache_page_bytes(dims)
    rc = lib().mla_append_latent(ctypes.byref(dims), _ptr(h), h.shape[0], _ptr(seq_idx), _ptr(pos), _ptr(W_dkv),
                                 _ptr(W_kr), _ptr(page_table), page_table.shape[0], page_table.shape[1],
                                 _ptr(cache_pool), num_pages, _ptr(workspace),
                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mla_append_latent")


def mla_append_latent_noalloc(dims, h, seq_idx, pos, W_dkv, W_kr, page_table, cache_pool, stream=None):
    """S1 without a workspace, for callers that cannot allocate device memory
    at call time: the library's fixed scratch array is used instead (65,536
    floats; an FP8-cache call needs n_tokens * d_c of them, bf16 and fp32
    caches none)."""
    _cuda(h, seq_idx, pos, W_dkv, W_kr, page_table, cache_pool)
    num_pages = cache_pool.numel() * cache_pool.element_size() // cache_page_bytes(dims)
    rc = lib().mla_append_latent_noalloc(ctypes.byref(dims), _ptr(h), h.shape[0], _ptr(seq_idx), _ptr(pos),
                                         _ptr(W_dkv), _ptr(W_kr), _ptr(page_table), page_table.shape[0],
                                         page_table.shape[1], _ptr(cache_pool), num_pages, _stream(stream))
    _check(rc, "mla_append_latent_noalloc")


def mla_decode(dims, q_nope, q_rope, W_uk, cache_pool, page_table, seq_lens, workspace, num_splits=0,
               stream=None):
    """S2+S3: absorb q and attend over the cache; partials go to workspace."""
    _cuda(q_nope, q_rope, W_uk, cache_pool, page_table, seq_lens, workspace)
    B, T = q_nope.shape[0], q_nope.shape[1]
    num_pages = cache_pool.numel() * cache_pool.element_size() // cache_page_bytes(dims)
    rc = lib().mla_decode(ctypes.byref(dims), _ptr(q_nope), _ptr(q_rope), _ptr(W_uk), _ptr(cache_pool), num_pages,
                          _ptr(page_table), page_table.shape[1], _ptr(seq_lens), B, T, num_splits,
                          _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "mla_decode")


def mla_combine(dims, W_uv, batch, n_q, workspace, out, lse_out=None, num_splits=0, stream=None):
    """S4: merge splits and apply W_uv; writes out [batch, n_q, n_h, d_v] and lse_out."""
    _cuda(W_uv, workspace, out, lse_out)
    rc = lib().mla_combine(ctypes.byref(dims), _ptr(W_uv), batch, n_q, num_splits, _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse_out),
                           _stream(stream))
    _check(rc, "mla_combine")


def prefill_workspace_bytes(dims: MlaDims, max_seq_len: int) -> int:
    return int(lib().mla_prefill_workspace_bytes(ctypes.byref(dims), max_seq_len))


def mla_prefill(dims, q_nope, q_rope, W_uk, W_uv, cache_pool, page_table, seq_lens, max_seq_len, workspace, out,
                lse_out=None, stream=None):
    """Prefill attention (non-absorbed form) of the n_q new tokens of each
    sequence, already appended: writes out [B, n_q, n_h, d_v] and lse_out."""
    _cuda(q_nope, q_rope, W_uk, W_uv, cache_pool, page_table, seq_lens, workspace, out, lse_out)
    B, T = q_nope.shape[0], q_nope.shape[1]
    num_pages = cache_pool.numel() * cache_pool.element_size() // cache_page_bytes(dims)
    rc = lib().mla_prefill(ctypes.byref(dims), _ptr(q_nope), _ptr(q_rope), _ptr(W_uk), _ptr(W_uv), _ptr(cache_pool),
                           num_pages, _ptr(page_table), page_table.shape[1], _ptr(seq_lens), B, T, max_seq_len,
                           _ptr(workspace), workspace.numel() * workspace.element_size(), _ptr(out), _ptr(lse_out),
                           _stream(stream))
    _check(rc, "mla_prefill")


def mla_get_status(stream=None) -> int:
    """Synchronise the stream and read/clear the device status word."""
    v = ctypes.c_int(0)
    _check(lib().mla_get_status(_stream(stream), ctypes.byref(v)), "mla_get_status")
    return v.value


def mla_set_trace_events(events):
    """Install torch.cuda.Event objects (2 per traced kernel, TRACE_KERNELS
    order, created with enable_timing=True) or None to uninstall."""
    if events is None:
        _check(lib().mla_set_trace_events(None, 0), "mla_set_trace_events")
        return
    for e in events:  # torch creates the CUDA event lazily, on first record
        if not e.cuda_event:
            e.record()
    arr = (ctypes.c_void_p * len(events))(*[ctypes.c_void_p(e.cuda_event) for e in events])
    _check(lib().mla_set_trace_events(arr, len(events)), "mla_set_trace_events")


def mla_set_timeline(buffer):
    """Install a device int64 tensor of 2 * len(TRACE_KERNELS) elements as the
    kernels' timeline (None switches it off).  Per kernel k, element 2k gets
    the earliest ns time a CTA passed its dependency wait (initialise to -1,
    i.e. all bits set) and 2k+1 the latest time a CTA finished (initialise to 0)."""
    if buffer is None:
        _check(lib().mla_set_timeline(None), "mla_set_timeline")
        return
    _cuda(buffer)
    if buffer.dtype != torch.int64 or buffer.numel() < 2 * len(TRACE_KERNELS):
        raise ValueError("timeline buffer: int64 tensor of 2 * len(TRACE_KERNELS) elements")
    _check(lib().mla_set_timeline(_ptr(buffer)), "mla_set_timeline")


def timeline_init(buffer):
    """Reset a timeline buffer (on the current stream): begins to UINT64_MAX, ends to 0."""
    v = buffer.view(-1, 2)
    v[:, 0].fill_(-1)
    v[:, 1].zero_()


def timeline_spans_ns(host_values) -> dict:
    """kernel name -> span (ns) from a timeline read back to the host
    (int64 values; begins of kernels that did not run stay all-ones)."""
    out = {}
    for k, name in enumerate(TRACE_KERNELS):
        b = int(host_values[2 * k]) & 0xFFFFFFFFFFFFFFFF
        e = int(host_values[2 * k + 1])
        if b != 0xFFFFFFFFFFFFFFFF and e > 0:
            out[name] = e - b
    return out
