// mla_append_latent_noalloc: the latent append for callers that cannot
// allocate device memory when they call us (a plugin or callback whose host
// framework owns all device memory and hands out no scratch buffer, or a loop
// where an allocation would synchronise the device).  Its scratch -- for an
// FP8 cache, the fp32 latent projections [n_tokens][d_c] that the projection
// kernel hands to the quantiser; bf16 and fp32 caches need none -- is a fixed
// array in this file instead of a caller workspace.
//
// The array lives in every GPU that loads the library, for as long as the
// process runs.  Calls share it: two calls whose kernels overlap on the GPU
// (on different streams, or different threads) race on it.  Nothing in it has
// to start at zero: the projection kernel writes every element the finalize
// kernel then reads, so stale contents from an earlier call are never used.
#include "mla_internal.cuh"

namespace mla {
int* device_status_word();
size_t cache_page_bytes(const mla_dims& d);
size_t append_scratch_floats(const mla_dims& d, int n_tokens);
}  // namespace mla

using namespace mla;

namespace {

// 65,536 floats (256 KiB): an FP8-cache append at DeepSeek-V3 dims (d_c = 512
// floats per token) of up to 128 tokens.
constexpr size_t kNoAllocScratchFloats = 65536;

static __device__ __align__(256) float g_noalloc_scratch[kNoAllocScratchFloats];

constexpr int kMaxDevices = 64;
float* g_scratch_addr[kMaxDevices] = {nullptr};

// Device address of the array on the current device, looked up once per device
// (host code must not pass the array's host-side name to a kernel).
float* scratch_on_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  if (!g_scratch_addr[dev]) {
    float* p = nullptr;
    if (cudaGetSymbolAddress((void**)&p, g_noalloc_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_addr[dev] = p;
  }
  return g_scratch_addr[dev];
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int mla_append_latent_noalloc(const mla_dims* dims, const void* h, int n_tokens, const int32_t* seq_idx,
                                         const int32_t* pos, const void* W_dkv, const void* W_kr,
                                         const int32_t* page_table, int batch, int max_pages, void* cache_pool,
                                         int num_pages, void* stream) {
  int rc = mla_check_dims(dims);
  if (rc != MLA_OK) return rc;
  if (n_tokens < 0 || batch < 1 || max_pages < 1 || num_pages < 1) return MLA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLA_OK;
  if (!h || !seq_idx || !pos || !W_dkv || !W_kr || !page_table || !cache_pool) return MLA_ERR_INVALID_ARG;
  // the scratch this request uses must fit the fixed array
  if (append_scratch_floats(*dims, n_tokens) > kNoAllocScratchFloats) return MLA_ERR_WORKSPACE;
  if (!aligned16(h) || !aligned16(W_dkv) || !aligned16(W_kr) || !aligned16(cache_pool)) return MLA_ERR_ALIGNMENT;
  float* scratch = scratch_on_current_device();
  if (!scratch) return MLA_ERR_CUDA;
  // scratch capacity 0 for the split-K partials: this entry point keeps the
  // kernels whose scratch is at most n_tokens * d_c floats
  cudaError_t e = launch_append(*dims, h, n_tokens, seq_idx, pos, W_dkv, W_kr, page_table, batch, max_pages,
                                cache_pool, num_pages, cache_page_bytes(*dims), scratch, 0, device_status_word(),
                                (cudaStream_t)stream);
  return e == cudaSuccess ? MLA_OK : MLA_ERR_LAUNCH;
}
