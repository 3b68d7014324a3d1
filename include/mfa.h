/*
 * mfa.h -- C ABI of libmfa.so: Multi-Matrix Factorization Attention (MFA) at
 * decode, and the MFA low-rank query projection, on NVIDIA B200 (sm_100a).
 *
 * What the operations are (Step-3 page, "Key points -> Architecture"): each new
 * token has 64 query heads of dimension 256, produced from the 7168-wide hidden
 * state through a 2048-wide low-rank bottleneck, and all 64 heads attend over a
 * single shared key head and a single shared value head of dimension 256 held in
 * the KV cache. The pages print no formula; the operation implemented is
 *
 *     out[b,h,:] = softmax_t( softmax_scale * q[b,h,:] . K_b[t,:] ) V_b[t,:],   t < seq_lens[b]
 *
 * with optional lse[b,h] = log sum_t exp(softmax_scale * q[b,h,:] . K_b[t,:]).
 * An empty sequence (seq_lens[b] == 0) yields zeros and lse = -inf.
 * K_b/V_b come from a contiguous slab or through a page table (PagedAttention,
 * cited in the Step-3 page's references). The pages deploy attention in FP8 and
 * in BF16 (Step-3 page, "Key points -> Throughput" and "Ablations"): the cache
 * may be bf16 or FP8 E4M3 with per-tensor scales. Long contexts are split over
 * many CTAs and merged with a log-sum-exp combine (Flash-Decoding, cited on the
 * DeepSeek-V4 page's reference list).
 *
 * Conventions for every entry point:
 *  - All tensor data pointers are DEVICE pointers on the current CUDA device;
 *    the mfa_tensor descriptor structs themselves live in host memory and are
 *    only read during the call. The caller owns every buffer.
 *  - Strides are in ELEMENTS. The innermost (last) dimension must have stride 1.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and never synchronise the host.
 *  - The return value reports host-detectable errors (bad descriptor, unsupported
 *    shape, too small workspace) and launch errors. Errors the GPU detects
 *    (a page id outside the pool, a sequence length outside the cache) are
 *    recorded in a per-device status word read by mfa_read_status(); outputs of
 *    the affected call are then unspecified, but no access leaves the buffers
 *    described by the arguments.
 *  - H = 64 and head dim = 256 are fixed; other shapes return MFA_ERR_UNSUPPORTED.
 *  - Requires a device of compute capability 10.0 (B200); otherwise
 *    MFA_ERR_UNSUPPORTED.
 */
#ifndef MFA_H_
#define MFA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* mfa_stream_t; /* identical to cudaStream_t */

enum mfa_dtype { MFA_BF16 = 0, MFA_F32 = 1, MFA_FP8_E4M3 = 2, MFA_I32 = 3 };

enum mfa_status {
  MFA_OK = 0,
  MFA_ERR_INVALID_ARG = 1,  /* null pointer, wrong rank/dtype, inconsistent shapes, bad stride */
  MFA_ERR_UNSUPPORTED = 2,  /* valid request this build does not implement (shape, device) */
  MFA_ERR_CUDA = 3,         /* a CUDA runtime/driver call or a kernel launch failed */
  MFA_ERR_WORKSPACE = 4,    /* caller workspace missing or too small */
  MFA_ERR_BAD_INDEX = 5,    /* (status word) page id or sequence length out of range */
  MFA_ERR_TIMEOUT = 6       /* (status word) a bounded in-kernel wait gave up */
};

/* A strided view of device memory. ndim in [1, 4]; shape/stride beyond ndim are
 * ignored. Strides in elements; data aligned to at least 16 bytes. */
typedef struct {
  void* data;
  int32_t dtype;  /* enum mfa_dtype */
  int32_t ndim;
  int64_t shape[4];
  int64_t stride[4];
} mfa_tensor;

/*
 * MFA decode attention (the operation above).
 *
 *  q          [B, 64, 256] bf16. Head and batch strides multiples of 8 elements.
 *  k_cache    contiguous: [B, Lmax, 256]; paged: [num_pages, page_size, 256].
 *             dtype MFA_BF16 or MFA_FP8_E4M3, equal to kv_dtype. Token and
 *             batch/page strides must be multiples of 16 bytes.
 *  v_cache    same shape, strides and dtype as k_cache.
 *  page_table NULL for a contiguous cache. Otherwise [B, max_pages] int32:
 *             token t of sequence b is row t % page_size of page
 *             page_table[b][t / page_size]. page_size in {16, 32, 64, 128, 256}.
 *             Entries past ceil(seq_lens[b] / page_size) are never read.
 *  seq_lens   [B] int32 on the device. 0 <= seq_lens[b] <= Lmax (contiguous) or
 *             <= max_pages * page_size (paged). Rows past seq_lens[b] are never
 *             used, whatever they hold (NaN included).
 *  out        [B, 64, 256], MFA_BF16 or MFA_F32, any strides (d stride 1).
 *  softmax_scale  multiplies q.k (1/16 = 1/sqrt(256) in the Step-3 setting).
 *  kv_dtype   MFA_BF16 or MFA_FP8_E4M3 (then k_scale = v_scale = 1).
 *
 * Uses a per-device workspace that the library allocates on the first call on
 * each device (cudaMalloc; keep that first call outside stream capture) and
 * reuses afterwards; concurrent calls on different streams share it and must
 * use mfa_decode_attention_ex with their own workspaces instead.
 */
int mfa_decode_attention(const mfa_tensor* q, const mfa_tensor* k_cache,
                         const mfa_tensor* v_cache, const mfa_tensor* page_table,
                         const mfa_tensor* seq_lens, mfa_tensor* out, float softmax_scale,
                         int kv_dtype, mfa_stream_t stream);

/*
 * As mfa_decode_attention, plus:
 *  k_scale, v_scale  per-tensor dequantisation scales of an FP8 cache
 *                    (K = code * k_scale, V = code * v_scale); must be 1 for bf16.
 *  num_splits        0: balanced split of all (sequence, 128-token tile) work over
 *                    the GPU's SMs (the default). s > 0: every sequence is cut
 *                    into s nearly equal token ranges, each its own work unit.
 *  lse_out           NULL or [B, 64] f32: natural-log log-sum-exp of the scaled
 *                    scores (-inf for empty sequences).
 *  workspace         device memory of at least
 *                    mfa_decode_workspace_size(B, num_splits) bytes, 256-byte
 *                    aligned, owned by the caller. It needs no
 *                    initialisation and its contents between calls do not
 *                    matter (fresh, reused, or left by another call of any
 *                    shape): everything the call's second kernel reads from it
 *                    is written earlier in the same call. Calls that overlap
 *                    on the GPU must not share a workspace.
 * Splitting never changes which cached rows contribute; the split plan depends
 * only on seq_lens, num_splits and the SM count, never on the cache layout, so a
 * paged and a contiguous cache holding the same rows give bit-identical results.
 */
int mfa_decode_attention_ex(const mfa_tensor* q, const mfa_tensor* k_cache,
                            const mfa_tensor* v_cache, const mfa_tensor* page_table,
                            const mfa_tensor* seq_lens, mfa_tensor* out, float softmax_scale,
                            int kv_dtype, float k_scale, float v_scale, int num_splits,
                            mfa_tensor* lse_out, void* workspace, size_t workspace_bytes,
                            mfa_stream_t stream);

/*
 * Grouped-query decode attention (GQA), the comparison shape for MFA (Step-3
 * summary page, "Key points -> Ablations": MFA beats MLA and GQA in decode
 * latency; GQA itself is Ainslie et al., in the pages' reference lists). 64
 * query heads of dimension 128 form 2 groups of 32 consecutive heads; group g
 * has its own key head and value head of dimension 128, so a cached token costs
 * 2 x 2 x 128 bf16 = 1024 bytes, exactly MFA's one 256-wide key and value head:
 *
 *   out[b,h,:] = softmax_t(softmax_scale * q[b,h,:] . K_b[t,g,:]) V_b[t,g,:],
 *   g = h / 32, over t < seq_lens[b]   (lse_out as for MFA).
 *
 *  q          [B, 64, 128] bf16 (head and batch strides multiples of 8 elements).
 *  k_cache    contiguous [B, Lmax, 2, 128] or paged [num_pages, page_size, 2, 128],
 *             bf16; a token's two group rows adjacent (stride 128 elements, d
 *             stride 1); token and batch/page strides multiples of 16 bytes.
 *  v_cache    same shape and strides as k_cache.
 *  page_table, seq_lens, num_splits, lse_out, workspace, stream
 *             as for mfa_decode_attention_ex (workspace size:
 *             mfa_decode_workspace_size(B, num_splits)).
 *  out        [B, 64, 128], MFA_BF16 or MFA_F32, any strides (d stride 1).
 *  softmax_scale  1/sqrt(128) in the comparison setting.
 * It runs on the MFA kernels: group g's 128 dims occupy head dims 128 g ..
 * 128 g + 127 of the 256-wide products (zeros elsewhere), so it issues the same
 * tensor-core instructions and reads the same bytes per token as MFA.
 * Returns as mfa_decode_attention_ex; MFA_ERR_UNSUPPORTED for other shapes.
 */
int mfa_gqa_decode_attention(const mfa_tensor* q, const mfa_tensor* k_cache,
                             const mfa_tensor* v_cache, const mfa_tensor* page_table,
                             const mfa_tensor* seq_lens, mfa_tensor* out, float softmax_scale,
                             int num_splits, mfa_tensor* lse_out, void* workspace,
                             size_t workspace_bytes, mfa_stream_t stream);

/* Bytes of workspace mfa_decode_attention_ex needs for `batch` sequences on the
 * current device with the given num_splits. 0 on error. */
size_t mfa_decode_workspace_size(int batch, int num_splits);

/*
 * mfa_decode_attention_ex without a workspace argument and without any device
 * allocation. The pages have no counterpart to this entry point: it is for
 * callers that cannot allocate device memory when they call in -- for example
 * a host framework that owns every device allocation through its own pool, or
 * a latency-critical loop that must not pay cudaMalloc's cost and implicit
 * device synchronisation -- and that cannot hand over a workspace either.
 *
 * The split workspace is a fixed 24 MiB device array inside libmfa.so, held
 * on every device that loads the library until the process exits. Requests
 * whose mfa_decode_workspace_size(B, num_splits) exceeds 24 MiB are rejected
 * with MFA_ERR_WORKSPACE (on a 148-SM B200 the default balanced plan needs
 * about 18.6 MiB plus 8 bytes per sequence; with num_splits = s the need is
 * about 64.3 KiB per sequence and split).
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture. Every call on a device uses the same array, which keeps
 * the last call's contents; nothing in it needs to start at zero (each call
 * writes what it reads), but calls that overlap on the GPU (different streams,
 * or different host threads) race on it: serialise them.
 * Arguments, results and errors are otherwise those of mfa_decode_attention_ex.
 */
int mfa_decode_attention_noalloc(const mfa_tensor* q, const mfa_tensor* k_cache,
                                 const mfa_tensor* v_cache, const mfa_tensor* page_table,
                                 const mfa_tensor* seq_lens, mfa_tensor* out, float softmax_scale,
                                 int kv_dtype, float k_scale, float v_scale, int num_splits,
                                 mfa_tensor* lse_out, mfa_stream_t stream);

/*
 * MFA low-rank query projection (Step-3 page, "Queries pass through a 2048-dim
 * low-rank bottleneck"): q_out = (x * W_qa) * W_qb, no bias, norm or activation.
 *
 *  x      [B, Dm] bf16 (Dm = 7168 in Step-3), row stride multiple of 8 elements.
 *  w_qa   [Dm, R] bf16 row-major (R = 2048).
 *  w_qb   [R, N] bf16 row-major (N = 64 * 256 = 16384).
 *  q_out  [B, N] bf16 (viewable as [B, 64, 256] when N = 16384).
 * 1 <= B <= 128; Dm a multiple of 64, R and N multiples of 128, R <= 131072.
 * The latent x * W_qa is accumulated in fp32 and carried into the second product
 * at about 16 significant bits (a bf16 high part plus a bf16 residual); q_out is
 * rounded once, to bf16.
 * Uses a per-device cached workspace (allocated on the first call; see above).
 */
int mfa_query_proj(const mfa_tensor* x, const mfa_tensor* w_qa, const mfa_tensor* w_qb,
                   mfa_tensor* q_out, mfa_stream_t stream);

/*
 * The query projection followed by decode attention on its result, in one call
 * (Step-3 page: the queries of every decode token come out of the 2048-wide
 * bottleneck, then attend over the shared key/value heads):
 *   q_out = (x * W_qa) * W_qb            as mfa_query_proj_ex, q_out [B, 64 * 256]
 *   out   = attention(q_out viewed as [B, 64, 256], caches)   as mfa_decode_attention_ex
 * The projection writes q straight in the layout the attention reads, and the
 * attention kernel is launched with programmatic dependent launch: the
 * projection lets it launch only after every earlier kernel on the stream has
 * completed, so its CTAs plan and start streaming key/value tiles on the SMs
 * the projection's CTAs leave, and read q once the projection has completed.
 * workspace: mfa_qproj_decode_workspace_size(B, Dm, R, num_splits) bytes,
 * 256-byte aligned: the projection's workspace (its first 4 KB zero before the
 * first use, as for mfa_query_proj_ex) followed by the attention's. Arguments
 * and errors otherwise as the two calls; nothing is launched if either call's
 * arguments are rejected.
 */
int mfa_qproj_decode_attention(const mfa_tensor* x, const mfa_tensor* w_qa,
                               const mfa_tensor* w_qb, mfa_tensor* q_out,
                               const mfa_tensor* k_cache, const mfa_tensor* v_cache,
                               const mfa_tensor* page_table, const mfa_tensor* seq_lens,
                               mfa_tensor* out, float softmax_scale, int kv_dtype, float k_scale,
                               float v_scale, int num_splits, mfa_tensor* lse_out,
                               void* workspace, size_t workspace_bytes, mfa_stream_t stream);

/* Bytes of workspace mfa_qproj_decode_attention needs. 0 on error. */
size_t mfa_qproj_decode_workspace_size(int batch, int dm, int rank, int num_splits);

/* As mfa_query_proj with a caller workspace of at least
 * mfa_query_proj_workspace_size(B, Dm, R) bytes, 256-byte aligned, that must be
 * zero-filled before its first use; every call returns its counters (the first
 * 4 KB) to zero, and the rest needs no initialisation. With B <= 8 both
 * products run in one persistent kernel that fills its load ring with W_qb
 * tiles while the latent is formed. */
int mfa_query_proj_ex(const mfa_tensor* x, const mfa_tensor* w_qa, const mfa_tensor* w_qb,
                      mfa_tensor* q_out, void* workspace, size_t workspace_bytes,
                      mfa_stream_t stream);

size_t mfa_query_proj_workspace_size(int batch, int dm, int rank);

/*
 * New-token key/value projection and cache append. The Step-3 page (Key points
 * -> Architecture) gives every token one shared key head and one shared value
 * head of dimension 256 fed by the 7168-wide hidden state; it prints no W_k or
 * W_v, and the plain reading is k = x * W_k, v = x * W_v (no bias, norm or
 * positional transform). Each sequence b's new row is written at token index
 * positions[b] of its cache -- the row the next decode-attention call reads
 * once seq_lens[b] = positions[b] + 1.
 *
 *  x          [B, Dm] bf16 hidden states of the new tokens (row stride a multiple of 8).
 *  w_k, w_v   [Dm, 256] bf16 row-major.
 *  k_cache, v_cache  the caches of mfa_decode_attention (contiguous [B, Lmax, 256]
 *             or paged [num_pages, page_size, 256]), same shape and strides,
 *             dtype kv_dtype; a bf16 cache takes the nearest bf16 of the
 *             projected value, an E4M3 cache the E4M3 code nearest to
 *             value / k_scale (resp. v_scale), saturating to +-448.
 *  page_table [B, max_pages] int32 (device) or NULL for contiguous caches.
 *  positions  [B] int32 (device): the row of each sequence's new token.
 *  k_scale, v_scale  > 0; must be 1 for bf16 caches.
 *  workspace  at least mfa_kv_append_workspace_size(B, Dm) bytes, 256-byte
 *             aligned, no initialisation needed (it holds split-K partials).
 * 1 <= B <= 256; Dm a multiple of 64. The projection accumulates in fp32 (split
 * over the hidden dimension, partials summed in a fixed order, so results do
 * not depend on timing) and rounds once, on store. Two kernels on `stream`.
 * A position outside the cache or a page id outside [0, num_pages) is not
 * written and is reported later by mfa_read_status as MFA_ERR_BAD_INDEX.
 * Returns MFA_OK, MFA_ERR_INVALID_ARG, MFA_ERR_UNSUPPORTED, MFA_ERR_WORKSPACE
 * or MFA_ERR_CUDA (then nothing was launched, or a launch failed).
 */
int mfa_kv_append(const mfa_tensor* x, const mfa_tensor* w_k, const mfa_tensor* w_v,
                  mfa_tensor* k_cache, mfa_tensor* v_cache, const mfa_tensor* page_table,
                  const mfa_tensor* positions, int kv_dtype, float k_scale, float v_scale,
                  void* workspace, size_t workspace_bytes, mfa_stream_t stream);

size_t mfa_kv_append_workspace_size(int batch, int hidden);

/*
 * Output projection of the attention layer: y = o * W_o, o the attention
 * outputs of each token with its 64 heads x 256 concatenated ([B, 16384] in
 * Step-3, i.e. mfa_decode_attention's out viewed as [B, 64 * 256]), W_o
 * [16384, 7168] bf16 row-major back to the hidden size, no bias. The pages name
 * no W_o; this is the plain reading of an attention layer's output projection.
 *
 *  o    [B, K] bf16, w_o [K, N] bf16, y [B, N] bf16 (row strides multiples of 8).
 *  workspace  at least mfa_output_proj_workspace_size(B, K, N) bytes, 256-byte
 *             aligned, no initialisation needed (split-K partials).
 * 1 <= B <= 256; K a multiple of 64, N of 128. fp32 accumulation split over K,
 * partials summed in a fixed order, one rounding to bf16. Two kernels on `stream`.
 * Returns MFA_OK, MFA_ERR_INVALID_ARG, MFA_ERR_UNSUPPORTED, MFA_ERR_WORKSPACE or
 * MFA_ERR_CUDA.
 */
int mfa_output_proj(const mfa_tensor* o, const mfa_tensor* w_o, mfa_tensor* y, void* workspace,
                    size_t workspace_bytes, mfa_stream_t stream);

size_t mfa_output_proj_workspace_size(int batch, int k, int n);

/*
 * Log-sum-exp merge of attention results computed over disjoint key ranges of
 * the same sequences (Flash-Decoding's combine, cited on the DeepSeek-V4 page's
 * reference list). Part s holds, for each sequence b and head h, the output
 * O_s[b,h,:] normalised over its own key range and that range's lse_s[b,h]
 * (natural log; -inf for an empty range) -- exactly what mfa_decode_attention_ex
 * returns in `out` (f32) and `lse_out` for the tokens it was given. The merge is
 *
 *     lse* = max_s lse_s,  w_s = exp(lse_s - lse*),
 *     out[b,h,:] = sum_s w_s O_s[b,h,:] / sum_s w_s,  lse[b,h] = lse* + log sum_s w_s,
 *
 * i.e. the attention over the union of the ranges. It is the exchange step of a
 * sequence whose cache is split across GPUs: each rank attends over its own
 * range, the (O, lse) parts are gathered (NCCL), and the owner merges them here.
 *
 *  o_parts    [S, B, 64, 256] f32 (device), 16-byte aligned, all strides multiples of 4.
 *  lse_parts  [S, B, 64] f32 (device), head stride 1. Values finite or -inf.
 *  out        [B, 64, 256] bf16 (8-byte aligned) or f32 (16-byte aligned),
 *             strides multiples of 4.
 *  lse_out    [B, 64] f32 or NULL.
 * 1 <= S <= 2^20, 1 <= B <= 2^20. Parts are merged in index order (results do
 * not depend on timing). A part whose lse is -inf has no weight and its O is not
 * used (it may hold anything); if every part of (b, h) is empty, out = 0 and
 * lse = -inf, as for an empty sequence. One kernel on `stream`; out and lse_out
 * must not overlap the parts. Returns MFA_OK, MFA_ERR_INVALID_ARG,
 * MFA_ERR_UNSUPPORTED (head count or dim not 64 / 256; not a B200) or MFA_ERR_CUDA.
 */
int mfa_lse_merge(const mfa_tensor* o_parts, const mfa_tensor* lse_parts, mfa_tensor* out,
                  mfa_tensor* lse_out, mfa_stream_t stream);

/* Synchronises `stream`, then reads (and, if reset != 0, clears) the current
 * device's status word: MFA_OK or the first MFA_ERR_BAD_INDEX / MFA_ERR_TIMEOUT
 * a kernel recorded since the last reset. Returns MFA_OK or MFA_ERR_CUDA. */
int mfa_read_status(mfa_stream_t stream, int reset, int* status_out);

/*
 * Failure-path self-test (no counterpart on the pages; failure handling is this
 * library's own). Every wait inside the library's kernels is bounded: when one
 * runs out the kernel records MFA_ERR_TIMEOUT in the status word, skips the
 * work that depended on it and returns, so the context stays usable. This call
 * makes such a wait run out on purpose without any fault: it launches the
 * decode call's combine kernel alone, on `stream`, for one split sequence whose
 * partial outputs no attention kernel will ever publish (its flags live in a
 * small fixed device array of the library that nothing sets), with the waits
 * limited to wait_ns (1 .. 10^10). It allocates nothing. Returns MFA_OK once
 * launched (or MFA_ERR_INVALID_ARG / MFA_ERR_CUDA); the kernel then ends after
 * about wait_ns, and mfa_read_status reports MFA_ERR_TIMEOUT.
 */
int mfa_selftest_wait_timeout(unsigned long long wait_ns, mfa_stream_t stream);

/* Static, human-readable name of a status code. */
const char* mfa_error_string(int code);

/* Text of the CUDA error behind the most recent MFA_ERR_CUDA returned to this
 * host thread (a static string; "no CUDA error recorded" if there was none). */
const char* mfa_last_cuda_error_string(void);

/* Library version: major * 10000 + minor * 100 + patch. */
int mfa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MFA_H_ */
