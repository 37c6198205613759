// C ABI of libmla (see include/mla.h): argument validation, workspace layout
// and kernel dispatch.  Every entry point launches on the caller's stream and
// returns without synchronising (except mla_get_status).
#include <math.h>
#include <stdio.h>

#include "mla_internal.cuh"

namespace mla {
size_t cache_page_bytes(const mla_dims& d);
bool decode_simt_supported(const mla_dims& d);
int append_max_d_model(int act_dtype);
size_t append_scratch_floats(const mla_dims& d, int n_tokens);
int absorb_max_d_nope();
int combine_max_splits();
int combine_max_d_c(int act_dtype);
}  // namespace mla

using namespace mla;

namespace mla {
static cudaEvent_t g_trace[2 * MLA_TRACE_COUNT];
static bool g_trace_on = false;
static unsigned long long* g_timeline = nullptr;
unsigned long long* timeline_ptr() { return g_timeline; }
// Called only where no launch error is pending; a failed record is dropped
// (and cleared) so that it is never reported as a kernel launch failure.
void trace_record(int kernel, bool end, cudaStream_t st) {
  if (g_trace_on && cudaEventRecord(g_trace[2 * kernel + (end ? 1 : 0)], st) != cudaSuccess)
    (void)cudaGetLastError();
}
}  // namespace mla

// Device status word (one instance per device that loads the library).
static __device__ int g_mla_status;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMinTilesPerSplit = 4;
int* g_status_ptr[kMaxDevices] = {nullptr};

int* status_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

int num_sms() { return device_sm_count(); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_dims(const mla_dims* d) {
  if (!d) return MLA_ERR_INVALID_ARG;
  if (d->n_heads < 1 || d->d_c < 16 || d->d_c % 16 || d->d_rope < 0 || d->d_rope % 2 || d->d_nope < 1 ||
      d->d_v < 1 || d->d_model < 32 || d->d_model % 32 || d->page_size < 1)
    return MLA_ERR_INVALID_ARG;
  if (!(d->softmax_scale > 0.f) || !isfinite(d->softmax_scale) || !(d->rope_base > 0.f) || !isfinite(d->rope_base))
    return MLA_ERR_INVALID_ARG;
  if (d->act_dtype != MLA_F32 && d->act_dtype != MLA_BF16) return MLA_ERR_INVALID_ARG;
  if (d->cache_dtype != MLA_F32 && d->cache_dtype != MLA_BF16 && d->cache_dtype != MLA_FP8_E4M3)
    return MLA_ERR_INVALID_ARG;
  if (d->cache_dtype == MLA_F32 && d->act_dtype != MLA_F32) return MLA_ERR_UNSUPPORTED;
  if (d->cache_dtype == MLA_FP8_E4M3 && d->d_c % 128) return MLA_ERR_UNSUPPORTED;
  if (d->d_nope % 8 || d->d_v > 1024) return MLA_ERR_UNSUPPORTED;
  if (d->d_model > append_max_d_model(d->act_dtype)) return MLA_ERR_UNSUPPORTED;
  if (d->d_nope > absorb_max_d_nope() || d->d_c > combine_max_d_c(d->act_dtype)) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

int auto_splits(const mla_dims& d, int batch, int n_q) {
  (void)batch;
  const int sms = num_sms();
  if (!(d.flags & MLA_FLAG_FORCE_SIMT) && decode_tc_supported(d, n_q)) return decode_tc_auto_splits(sms, n_q);
  const int hg = d.n_heads % 8 == 0 && d.d_c / 16 <= 32 ? 8 : 4;
  const int per_split = n_q * (d.n_heads / hg);
  int w = (4 * sms + per_split - 1) / per_split;
  return w < 1 ? 1 : (w > combine_max_splits() ? combine_max_splits() : w);
}

int launch_status(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_LAUNCH; }

}  // namespace

namespace mla {
// Device status word of the current device, for entry points in other files.
int* device_status_word() { return status_ptr(); }
}  // namespace mla

extern "C" {

size_t mla_cache_page_bytes(const mla_dims* dims) {
  if (check_dims(dims) != MLA_OK) return 0;
  return cache_page_bytes(*dims);
}

int mla_check_dims(const mla_dims* dims) { return check_dims(dims); }

size_t mla_append_workspace_bytes(const mla_dims* dims, int n_tokens) {
  if (check_dims(dims) != MLA_OK || n_tokens < 0) return 0;
  return align_up(sizeof(float) * append_scratch_floats(*dims, n_tokens), 256);
}

size_t mla_append_workspace_bytes_fast(const mla_dims* dims, int n_tokens) {
  if (check_dims(dims) != MLA_OK || n_tokens < 0) return 0;
  const size_t need = mla_append_workspace_bytes(dims, n_tokens);
  const size_t fast = align_up(sizeof(float) * append_splitk_floats(*dims, n_tokens), 256);
  return fast > need ? fast : need;
}

int mla_append_latent(const mla_dims* dims, const void* h, int n_tokens, const int32_t* seq_idx,
                      const int32_t* pos, const void* W_dkv, const void* W_kr, const int32_t* page_table,
                      int batch, int max_pages, void* cache_pool, int num_pages, void* workspace,
                      size_t ws_bytes, void* stream) {
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (n_tokens < 0 || batch < 1 || max_pages < 1 || num_pages < 1) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!h || !seq_idx || !pos || !W_dkv || !W_kr || !page_table || !cache_pool) return MLA_ERR_INVALID_ARG;
  const size_t need = mla_append_workspace_bytes(dims, n_tokens);
  if (need > 0 && (!workspace || ws_bytes < need)) return MLA_ERR_WORKSPACE;
  if (!aligned16(h) || !aligned16(W_dkv) || !aligned16(W_kr) || !aligned16(cache_pool) ||
      (need > 0 && !aligned16(workspace)))
    return MLA_ERR_ALIGNMENT;
  return launch_status(launch_append(*dims, h, n_tokens, seq_idx, pos, W_dkv, W_kr, page_table, batch,
                                     max_pages, cache_pool, num_pages, cache_page_bytes(*dims),
                                     static_cast<float*>(workspace), workspace ? ws_bytes / sizeof(float) : 0,
                                     status_ptr(), (cudaStream_t)stream));
}

int mla_auto_splits(const mla_dims* dims, int batch, int n_q) {
  int rc = check_dims(dims);
  if (rc != MLA_OK) return -rc;
  if (batch < 1 || n_q < 1) return -MLA_ERR_INVALID_ARG;
  return auto_splits(*dims, batch, n_q);
}

size_t mla_decode_workspace_bytes(const mla_dims* dims, int batch, int n_q, int num_splits) {
  if (check_dims(dims) != MLA_OK || batch < 1 || n_q < 1 || num_splits < 0) return 0;
  const int W = num_splits > 0 ? num_splits : auto_splits(*dims, batch, n_q);
  return decode_layout(*dims, batch, n_q, W).total;
}

int mla_decode_path(const mla_dims* dims, int n_q) {
  int rc = check_dims(dims);
  if (rc != MLA_OK) return -rc;
  if (!(dims->flags & MLA_FLAG_FORCE_SIMT) && decode_tc_supported(*dims, n_q)) return 1;
  return decode_simt_supported(*dims) ? 0 : -MLA_ERR_UNSUPPORTED;
}

int mla_decode(const mla_dims* dims, const void* q_nope, const void* q_rope, const void* W_uk,
               const void* cache_pool, int num_pages, const int32_t* page_table, int max_pages,
               const int32_t* seq_lens, int batch, int n_q, int num_splits, void* workspace, size_t ws_bytes,
               void* stream) {
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (batch < 1 || n_q < 1 || num_pages < 1 || max_pages < 1 || num_splits < 0 ||
      num_splits > combine_max_splits())
    return MLA_ERR_INVALID_ARG;
  if (!q_nope || !q_rope || !W_uk || !cache_pool || !page_table || !seq_lens) return MLA_ERR_INVALID_ARG;
  const int path = mla_decode_path(dims, n_q);
  if (path < 0) return -path;
  // The workspace layout is the one of the requested (or automatic) split
  // count; with num_splits = 0 short contexts use fewer splits (at least
  // kMinTilesPerSplit key tiles each, counted on batch * max_pages), which the
  // plan records for mla_combine.
  const int W_layout = num_splits > 0 ? num_splits : auto_splits(*dims, batch, n_q);
  const DecodeLayout L = decode_layout(*dims, batch, n_q, W_layout);
  int W = W_layout;
  if (num_splits == 0) {
    const long long cap = ((long long)batch * max_pages + kMinTilesPerSplit - 1) / kMinTilesPerSplit;
    if (cap < W) W = (int)(cap > 0 ? cap : 1);
  }
  if (!workspace || ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (!aligned16(W_uk) || !aligned16(cache_pool) || !aligned16(workspace)) return MLA_ERR_ALIGNMENT;
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* plan = reinterpret_cast<int32_t*>(ws + L.off_plan);
  int* status = status_ptr();
  trace_record(MLA_TRACE_ABSORB, false, st);
  const int n_slots = batch + W - 1;
  const bool q_f16 = path == 1 && decode_tc_wants_f16_queries(*dims);
  cudaError_t e = launch_absorb_and_plan(*dims, q_nope, q_rope, W_uk, seq_lens, batch, n_q, max_pages, W, ws + L.off_q,
                                         q_f16, plan, reinterpret_cast<float*>(ws + L.off_lse),
                                         (size_t)n_q * n_slots * dims->n_heads, status, st);
  trace_record(MLA_TRACE_ABSORB, true, st);
  if (e != cudaSuccess) return MLA_ERR_LAUNCH;
  DecodeParams p;
  p.d = *dims;
  p.q_abs = ws + L.off_q;
  p.pool = static_cast<const uint8_t*>(cache_pool);
  p.page_bytes = cache_page_bytes(*dims);
  p.num_pages = num_pages;
  p.page_table = page_table;
  p.max_pages = max_pages;
  p.seq_lens = seq_lens;
  p.plan = plan;
  p.o_part = reinterpret_cast<float*>(ws + L.off_o);
  p.lse_part = reinterpret_cast<float*>(ws + L.off_lse);
  p.batch = batch;
  p.n_q = n_q;
  p.splits = W;
  p.n_slots = n_slots;
  p.scale_log2 = dims->softmax_scale * kLog2e;
  p.status = status;
  p.timeline = timeline_ptr();
  trace_record(MLA_TRACE_ATTEND, false, st);
  e = path == 1 ? launch_decode_tc(p, st) : launch_decode_simt(p, st);
  trace_record(MLA_TRACE_ATTEND, true, st);
  return launch_status(e);
}

int mla_combine(const mla_dims* dims, const void* W_uv, int batch, int n_q, int num_splits, const void* workspace,
                size_t ws_bytes, void* out, float* lse_out, void* stream) {
  int rc = check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (batch < 1 || n_q < 1 || num_splits < 0) return MLA_ERR_INVALID_ARG;
  if (!W_uv || !out) return MLA_ERR_INVALID_ARG;
  const int W = num_splits > 0 ? num_splits : auto_splits(*dims, batch, n_q);
  const DecodeLayout L = decode_layout(*dims, batch, n_q, W);
  if (!workspace || ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  if (!aligned16(W_uv) || !aligned16(workspace)) return MLA_ERR_ALIGNMENT;
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  trace_record(MLA_TRACE_COMBINE, false, (cudaStream_t)stream);
  // the partials' row type follows the decode path that wrote them
  const bool part_bf16 = mla_decode_path(dims, n_q) == 1;
  cudaError_t e = launch_combine(*dims, W_uv, batch, n_q, reinterpret_cast<const int32_t*>(ws + L.off_plan),
                                 reinterpret_cast<const float*>(ws + L.off_o), part_bf16,
                                 reinterpret_cast<const float*>(ws + L.off_lse), out, lse_out, status_ptr(),
                                 (cudaStream_t)stream);
  trace_record(MLA_TRACE_COMBINE, true, (cudaStream_t)stream);
  return launch_status(e);
}

int mla_set_trace_events(void* const* events, int n_events) {
  if (!events) {
    g_trace_on = false;
    return MLA_OK;
  }
  if (n_events < 2 * MLA_TRACE_COUNT) return MLA_ERR_INVALID_ARG;
  for (int i = 0; i < 2 * MLA_TRACE_COUNT; ++i) g_trace[i] = (cudaEvent_t)events[i];
  g_trace_on = true;
  return MLA_OK;
}

int mla_set_timeline(unsigned long long* device_buffer) {
  g_timeline = device_buffer;
  return MLA_OK;
}

int mla_get_status(void* stream, int* status) {
  if (!status) return MLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_mla_status, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_mla_status, &zero, sizeof(int)) != cudaSuccess) return MLA_ERR_CUDA;
  *status = v;
  return MLA_OK;
}

const char* mla_error_string(int code) {
  switch (code) {
    case MLA_OK: return "ok";
    case MLA_ERR_INVALID_ARG: return "invalid argument";
    case MLA_ERR_UNSUPPORTED: return "unsupported dims or dtypes";
    case MLA_ERR_WORKSPACE: return "workspace missing or too small";
    case MLA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case MLA_ERR_LAUNCH: return "kernel launch failed";
    case MLA_ERR_TIMEOUT: return "bounded wait expired on the device";
    case MLA_ERR_BOUNDS: return "page index, position or sequence length out of range";
    case MLA_ERR_CUDA: return "CUDA runtime call failed";
    default: return "unknown error";
  }
}

}  // extern "C"
