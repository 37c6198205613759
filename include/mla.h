/*
 * mla.h - C ABI of libmla: Multi-Head Latent Attention (MLA) decode on a paged
 * latent cache, absorbed form, for NVIDIA B200 (sm_100a).
 *
 * The operation is the decode step of "DeepSeek MLA Architecture: How
 * Multi-Head Latent Attention Cuts KV Cache by 93%" (explore.n1n.ai):
 *   - each token caches only c = W^DKV h (d_c scalars, "1. Low-Rank Key-Value
 *     Compression") and one shared, pre-rotated RoPE key k^R = RoPE(W^KR h)
 *     (d_rope scalars, "3. Decoupled RoPE and Matrix Absorption");
 *   - a query is absorbed into latent space, q~_h = (W^UK_h)^T q^C_h, and
 *     scored directly against the cached rows: score = q~_h . c_s + q^R_h . k^R_s
 *     ("3. Decoupled RoPE and Matrix Absorption", eq. for q~ and the split
 *     score), scaled by 1/sqrt(d_nope + d_rope);
 *   - the softmax-weighted latent sum u_h = sum_s p_s c_s is formed in latent
 *     space and W^UV_h is applied afterwards, o_h = W^UV_h u_h.
 * The page's single-token decoding module appends the step's token and then
 * attends; this library splits that step into three calls (append, decode,
 * combine) over a caller-owned paged cache.
 *
 * General conventions
 *   - Every pointer argument is a DEVICE pointer owned by the caller unless
 *     stated otherwise.  The library allocates no device memory: scratch is the
 *     caller's `workspace`, sized by the matching *_workspace_bytes() call,
 *     except for mla_append_latent_noalloc, whose scratch is a fixed 256 KiB
 *     array inside the library on every GPU that loads it (see its note).
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL
 *     is the legacy default stream).  Nothing synchronises except
 *     mla_get_status().  Kernels run on the current CUDA device.
 *   - Return value: MLA_OK, or an MLA_ERR_* code for errors the host can see
 *     (bad arguments, unsupported shapes, small workspace, misalignment, a
 *     failed launch).  Errors that depend on device-resident values (an
 *     out-of-range page index, a sequence shorter than n_q) are recorded in a
 *     device status word; the offending row or work item is skipped, and
 *     mla_get_status() reports the code.
 *   - Row-major layouts; "[a, b, c]" lists dimensions outermost first.
 *   - Tensors of "act" type are float32 (MLA_F32) or bfloat16 (MLA_BF16)
 *     according to mla_dims.act_dtype.
 *
 * Paged cache layout (`cache_pool`, num_pages pages of page_size tokens):
 *   MLA_F32 / MLA_BF16 cache: page = [page_size][d_c + d_rope] rows of that
 *     type; a row is [c (d_c) | k^R (d_rope)].  bf16 V3 dims: 1152 B per row.
 *   MLA_FP8_E4M3 cache: page = [page_size][d_c] e4m3 codes of c, then
 *     [page_size][d_rope] bf16 k^R, then [page_size][d_c/128] fp32 scales;
 *     c[j] = e4m3(code[j]) * scale[j/128], scale = amax of the 128-wide tile
 *     / 448 (1 for an all-zero tile).  Sub-blocks start at multiples of 128 B.
 *   mla_cache_page_bytes() gives the page size in bytes.
 *   Token `pos` of sequence b lives in row pos % page_size of physical page
 *   page_table[b * max_pages + pos / page_size].
 */
#ifndef MLA_H_
#define MLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MLA_F32 = 0, MLA_BF16 = 1, MLA_FP8_E4M3 = 2 } mla_dtype;

enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1, /* null pointer, negative size, inconsistent dims */
  MLA_ERR_UNSUPPORTED = 2, /* dims/dtypes with no kernel */
  MLA_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than required */
  MLA_ERR_ALIGNMENT = 4,   /* a pointer not 16-byte aligned */
  MLA_ERR_LAUNCH = 5,      /* a kernel launch failed (cudaGetLastError) */
  MLA_ERR_TIMEOUT = 6,     /* device: a bounded wait in a kernel gave up */
  MLA_ERR_BOUNDS = 7,      /* device: page index / position / length out of range */
  MLA_ERR_CUDA = 8         /* a CUDA runtime call failed */
};

/* mla_dims.flags */
#define MLA_FLAG_FORCE_SIMT 1u /* use the CUDA-core kernels even where tcgen05 kernels exist */
/* Self-test of failure detection, for the tensor-core kernels at DeepSeek-V3
 * dims (bf16 activations):
 *   - mla_decode: the attention kernel's load producers issue no loads, so the
 *     MMA issuers' and softmax warps' bounded waits (~2 s) expire; the CTA
 *     pair that gives up first tells its peer, every role stops, the kernel
 *     waits (bounded) for the MMAs it issued and frees its tensor memory;
 *     MLA_ERR_TIMEOUT is recorded and the split partials are not valid.
 *   - mla_combine: the kernel does not fetch its weights, so its bounded wait
 *     for them expires; MLA_ERR_TIMEOUT is recorded and out and lse_out are
 *     left unwritten.
 *   - mla_prefill: the up-projection GEMM's and the attention kernel's load
 *     producers issue no loads; both kernels' waits expire (~2 s each), each
 *     CTA waits (bounded) for the MMAs it issued and frees its tensor memory;
 *     MLA_ERR_TIMEOUT is recorded and out / lse_out are not valid.
 *   - mla_append_latent on its tensor-core GEMM paths (16 or more tokens with
 *     the fast workspace, or 512 or more): the GEMM's producer issues no
 *     loads and its wait expires the same way; MLA_ERR_TIMEOUT is recorded
 *     and the step's cache rows are not valid (a later append rewrites them).
 * No copy is in flight when a wait gives up, and the context stays usable.
 * Ignored by the other kernels. */
#define MLA_FLAG_SELFTEST_STALL 2u

typedef struct {
  int32_t n_heads;     /* n_h (128 for DeepSeek-V3) */
  int32_t d_c;         /* latent rank (512); multiple of 16; multiple of 128 for FP8 */
  int32_t d_rope;      /* decoupled RoPE width (64); even */
  int32_t d_nope;      /* per-head content query/key width (128) */
  int32_t d_v;         /* per-head value width (128) */
  int32_t d_model;     /* model width d (7168); multiple of 8 */
  int32_t page_size;   /* tokens per cache page (64) */
  int32_t act_dtype;   /* mla_dtype: MLA_F32 or MLA_BF16 */
  int32_t cache_dtype; /* mla_dtype: MLA_F32 (needs act F32), MLA_BF16 or MLA_FP8_E4M3 (need act BF16) */
  float softmax_scale; /* 1/sqrt(d_nope + d_rope) in the pages' module */
  float rope_base;     /* 10000 */
  uint32_t flags;      /* MLA_FLAG_* */
} mla_dims;

/* Bytes of one cache page (host only, no GPU needed). 0 if dims are invalid. */
size_t mla_cache_page_bytes(const mla_dims* dims);

/* Host-side validation of dims (no GPU needed): MLA_OK or an error code. */
int mla_check_dims(const mla_dims* dims);

/* ---------------------------------------------------------------------------
 * S1  mla_append_latent: write the latent rows of n_tokens new tokens.
 *   c_n = W_dkv h_n                    ("1. Low-Rank Key-Value Compression")
 *   k^R_n = RoPE(W_kr h_n, pos[n])     ("3. Decoupled RoPE and Matrix Absorption";
 *                                       rotate-half RoPE of the decoding module,
 *                                       angle pos * rope_base^(-i/(d_rope/2)))
 * and store [c_n | k^R_n] at (seq_idx[n], pos[n]) of the paged cache, rounded
 * to the cache type (fp32 accumulation; RNE to bf16; FP8 per the layout above).
 *   h          [n_tokens, d_model] act
 *   seq_idx    [n_tokens] int32, sequence of each token, in [0, batch)
 *   pos        [n_tokens] int32, position of each token, >= 0
 *   W_dkv      [d_c, d_model] act;  W_kr [d_rope, d_model] act
 *   page_table [batch, max_pages] int32
 *   cache_pool num_pages pages (layout above), written
 *   workspace  >= mla_append_workspace_bytes(dims, n_tokens) bytes of scratch
 *              (fp32 c values between the projection and the FP8 quantiser;
 *              0 bytes, and workspace may be NULL, for fp32/bf16 caches).
 *              With >= mla_append_workspace_bytes_fast(dims, n_tokens) bytes
 *              (16-byte aligned), a step of 16 to 511 tokens at DeepSeek-V3
 *              dims with bf16 activations takes the split-K tensor-core
 *              projection, whose fp32 partial tiles live there; with less it
 *              takes the cluster kernel.  Same results up to fp32 summation
 *              order.
 * d_model must be a multiple of 32 and <= 8192 (bf16) / 4096 (fp32): the
 * projection keeps a lane's slice of each weight row in registers
 * (MLA_ERR_UNSUPPORTED otherwise).
 * Out-of-range seq_idx/pos/page entries: the token is skipped and
 * MLA_ERR_BOUNDS is recorded in the device status word.  n_tokens == 0 is a no-op.
 * ------------------------------------------------------------------------- */
size_t mla_append_workspace_bytes(const mla_dims* dims, int n_tokens);
/* The workspace that enables the fastest append path for this request (never
 * less than mla_append_workspace_bytes); 0 on invalid dims. */
size_t mla_append_workspace_bytes_fast(const mla_dims* dims, int n_tokens);
/* mla_append_latent_noalloc: mla_append_latent for callers that cannot
 * allocate device memory at call time (a plugin or callback whose host
 * framework owns all device memory and offers no scratch buffer, or a loop in
 * which an allocation would synchronise the device).  The source articles have no
 * counterpart: this is a deployment variant of the S1 append.
 * Same arguments and results as mla_append_latent, without the workspace: the
 * fp32 scratch lives in a fixed array inside the library, 65,536 floats
 * (256 KiB) on every GPU that loads it, held until the process exits.
 *   - The scratch a call uses is what mla_append_workspace_bytes() reports:
 *     n_tokens * d_c floats for an FP8 cache, none for bf16 and fp32 caches.
 *     An FP8 request must fit the array (n_tokens * d_c <= 65536: 128 tokens
 *     at DeepSeek-V3 dims); a larger one returns MLA_ERR_WORKSPACE and
 *     launches nothing.  bf16 and fp32 caches have no size limit here.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *   - All calls share the array: calls whose kernels overlap on the GPU race.
 *     Nothing in it needs clearing between calls.
 *   - It calls no cudaMalloc/cudaFree and no allocating library routine. */
int mla_append_latent_noalloc(const mla_dims* dims, const void* h, int n_tokens,
                              const int32_t* seq_idx, const int32_t* pos,
                              const void* W_dkv, const void* W_kr,
                              const int32_t* page_table, int batch, int max_pages,
                              void* cache_pool, int num_pages, void* stream);

int mla_append_latent(const mla_dims* dims, const void* h, int n_tokens,
                      const int32_t* seq_idx, const int32_t* pos,
                      const void* W_dkv, const void* W_kr,
                      const int32_t* page_table, int batch, int max_pages,
                      void* cache_pool, int num_pages,
                      void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * S2+S3  mla_decode: absorb the queries and run split-KV attention over the
 * cache, leaving per-split partial results in `workspace` for mla_combine.
 *   For sequence b, query j (position p = seq_lens[b] - n_q + j), head h:
 *     q~ = W_uk[h]^T q_nope[b,j,h]             (absorption, eq. for q~)
 *     q^R = RoPE(q_rope[b,j,h], p)
 *     a_s = softmax_scale * (q~ . c_s + q^R . k^R_s),   s = 0 .. p
 *   and, per split of the keys, the normalised latent aggregate
 *   u = sum_s softmax(a)_s c_s with its log-sum-exp.
 * The query j of a sequence sees keys 0..p: causal among the n_q new tokens,
 * which must already be in the cache (append first, then attend).
 *   q_nope     [batch, n_q, n_heads, d_nope] act
 *   q_rope     [batch, n_q, n_heads, d_rope] act, NOT rotated
 *   W_uk       [n_heads, d_nope, d_c] act
 *   cache_pool, num_pages, page_table [batch, max_pages], as above (read only)
 *   seq_lens   [batch] int32, tokens in the cache per sequence (>= n_q)
 *   num_splits number of key-range splits shared by all sequences; 0 = auto
 *   workspace  >= mla_decode_workspace_bytes(dims, batch, n_q, num_splits)
 * The workspace is consumed by the next mla_combine with the same dims, batch,
 * n_q and num_splits.
 * ------------------------------------------------------------------------- */
size_t mla_decode_workspace_bytes(const mla_dims* dims, int batch, int n_q, int num_splits);
int mla_decode(const mla_dims* dims, const void* q_nope, const void* q_rope,
               const void* W_uk, const void* cache_pool, int num_pages,
               const int32_t* page_table, int max_pages, const int32_t* seq_lens,
               int batch, int n_q, int num_splits,
               void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * S4  mla_combine: merge the splits and apply the value up-projection.
 *   u = sum_i exp(lse_i - LSE) u_i,  LSE = log sum_i exp(lse_i)
 *   o_h = W_uv[h] u_h  ("value aggregation ... directly against c", with W^UV
 *                       applied after the softmax, as in the decoding module)
 *   W_uv    [n_heads, d_v, d_c] act
 *   out     [batch, n_q, n_heads, d_v] act, written
 *   lse_out [batch, n_q, n_heads] float32 natural-log softmax denominators of
 *           the scaled scores, written; may be NULL
 * `workspace`, `batch`, `n_q`, `num_splits` as passed to the mla_decode call
 * whose results are combined.
 * ------------------------------------------------------------------------- */
int mla_combine(const mla_dims* dims, const void* W_uv, int batch, int n_q, int num_splits,
                const void* workspace, size_t ws_bytes, void* out, float* lse_out,
                void* stream);

/* ---------------------------------------------------------------------------
 * Prefill (many new tokens per sequence)  mla_prefill: the non-absorbed form.
 * A prefill step is compute-bound, and there reconstructing each head's keys
 * and values from the latent is cheaper than the absorbed form ("DeepSeek MLA
 * Architecture: How Multi-Head Latent Attention Cuts KV Cache by 93%",
 * opening section on the prefill and decode phases; "1. Low-Rank Key-Value
 * Compression"; "3. Decoupled RoPE and Matrix Absorption").  For sequence b,
 * query j (position p = seq_lens[b] - n_q + j), head h, keys s = 0 .. p:
 *   k_{s,h} = [W_uk[h] c_s ; k^R_s],  v_{s,h} = W_uv[h] c_s,
 *   o_h = softmax(softmax_scale * [q_nope ; RoPE(q_rope, p)] . k_{s,h}) v_{s,h}
 * which is the same result mla_decode + mla_combine give (causal among the
 * n_q new tokens, which must already be in the cache).
 *   q_nope, q_rope, W_uk, cache_pool, num_pages, page_table, max_pages,
 *   seq_lens, batch, n_q as for mla_decode; W_uv as for mla_combine
 *   max_seq_len  host-side upper bound of seq_lens[b] (sizes the grids and the
 *                workspace); a longer sequence is skipped and MLA_ERR_BOUNDS
 *                recorded
 *   workspace    >= mla_prefill_workspace_bytes(dims, max_seq_len): one
 *                sequence's gathered latent rows, its per-head keys and
 *                values and its rotated queries (about 113 KB per token of
 *                max_seq_len at DeepSeek-V3 dims); sequences run one after
 *                another
 *   out          16-byte aligned (MLA_ERR_ALIGNMENT otherwise)
 *   out [batch, n_q, n_heads, d_v] act, lse_out [batch, n_q, n_heads] float32
 *   natural-log softmax denominators (may be NULL)
 * DeepSeek-V3 dims only (d_c 512, d_rope 64, d_nope = d_v = 128, 64-token
 * pages), bf16 activations, bf16 or FP8 cache; MLA_ERR_UNSUPPORTED otherwise.
 * ------------------------------------------------------------------------- */
size_t mla_prefill_workspace_bytes(const mla_dims* dims, int max_seq_len);
int mla_prefill(const mla_dims* dims, const void* q_nope, const void* q_rope,
                const void* W_uk, const void* W_uv, const void* cache_pool, int num_pages,
                const int32_t* page_table, int max_pages, const int32_t* seq_lens,
                int batch, int n_q, int max_seq_len, void* workspace, size_t ws_bytes,
                void* out, float* lse_out, void* stream);

/* Which decode kernel mla_decode would launch for these dims on the current
 * device: 0 = CUDA-core (SIMT) kernel, 1 = tcgen05 kernel; <0 = error code. */
int mla_decode_path(const mla_dims* dims, int n_q);

/* Number of key-range splits that num_splits = 0 selects on the current device. */
int mla_auto_splits(const mla_dims* dims, int batch, int n_q);

/* Tracing.  Kernels of the calls above, in launch order per step: */
enum {
  MLA_TRACE_APPEND_PROJECT = 0, /* mla_append_latent: [W_dkv; W_kr] h, RoPE, paged store */
  MLA_TRACE_APPEND_FINALIZE = 1,/* mla_append_latent: FP8 quantiser (FP8 caches only) */
  MLA_TRACE_ABSORB = 2,         /* mla_decode: q~ = W_uk^T q_nope, RoPE(q_rope), split plan */
  MLA_TRACE_ATTEND = 3,         /* mla_decode: split-KV attention over the cache */
  MLA_TRACE_COMBINE = 4,        /* mla_combine: split merge and W_uv */
  MLA_TRACE_PREFILL_PREP = 5,   /* mla_prefill: query assembly (RoPE) and latent gather */
  MLA_TRACE_PREFILL_UPPROJ = 6, /* mla_prefill: per-head keys and values from the latent */
  MLA_TRACE_PREFILL_ATTEND = 7, /* mla_prefill: causal attention */
  MLA_TRACE_COUNT = 8
};
/* Install a table of 2*MLA_TRACE_COUNT cudaEvent_t (passed as void*, created
 * by the caller with timing enabled): later calls record events[2k] before and
 * events[2k+1] after kernel k on the launch stream (both back to back when
 * the call launches no kernel k).  NULL uninstalls.  The
 * table is process-wide host state read at launch time; it is not
 * thread-safe.  Returns MLA_OK or MLA_ERR_INVALID_ARG (n_events too small). */
int mla_set_trace_events(void* const* events, int n_events);

/* Device timeline of the kernels, for timing a step from CUDA-graph replays
 * (where events recorded between kernels would break their programmatic
 * dependent launch).  `device_buffer` is a DEVICE array of 2*MLA_TRACE_COUNT
 * uint64 owned by the caller, or NULL to switch the timeline off.  Kernels
 * launched while it is installed write, for each kernel k above:
 *   [2k]   the earliest %globaltimer value (ns) at which one of its CTAs had
 *          passed its wait for the preceding kernel (atomic minimum: the
 *          caller initialises it to UINT64_MAX),
 *   [2k+1] the latest value at which one of its CTAs finished (atomic
 *          maximum: initialised to 0).
 * So [2k+1] - [2k] is kernel k's span on the device with its dependency
 * already met.  The pointer is read at launch time (a graph keeps the value it
 * was captured with); it is process-wide host state and not thread-safe.
 * Returns MLA_OK. */
int mla_set_timeline(unsigned long long* device_buffer);

/* Synchronise `stream`, then read and clear the device status word of the
 * current device into *status (MLA_OK or MLA_ERR_TIMEOUT / MLA_ERR_BOUNDS).
 * Returns MLA_OK, or MLA_ERR_CUDA if the synchronisation failed. */
int mla_get_status(void* stream, int* status);

/* Static description of an error code (never NULL). */
const char* mla_error_string(int code);

#ifdef __cplusplus
}
#endif
#endif /* MLA_H_ */
