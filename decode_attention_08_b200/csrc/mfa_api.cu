// mfa_api.cu -- the extern "C" entry points of libmfa.so (declared in
// include/mfa.h): argument validation, TMA tensor-map encoding, workspace
// management and kernel launches. No computation happens here.

#include <cstdio>
#include <cstring>
#include <initializer_list>
#include <mutex>

#include "../../include/mfa.h"
#include "mfa_internal.h"

namespace mfa {
int decode_smem_bytes();
cudaError_t launch_combine_only(const DecodeParams& p, cudaStream_t stream);
cudaError_t launch_decode(bool paged, bool fp8, const CUtensorMap& tq, const CUtensorMap& tk,
                          const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream);
int qproj_smem_bytes(int n_cols);
bool qproj_fused_fits(int n1, int n2, int k2_blocks);
cudaError_t launch_qproj_fused(const CUtensorMap& twa, const CUtensorMap& tx,
                               const CUtensorMap& twb, const CUtensorMap& tl,
                               const QprojFusedParams& p, int grid, cudaStream_t stream);
cudaError_t launch_qproj(const CUtensorMap& tw, const CUtensorMap& ta, const QprojParams& p,
                         int m_tiles, cudaStream_t stream);
cudaError_t launch_kv_append(const CUtensorMap& twk, const CUtensorMap& twv, const CUtensorMap& tx,
                             const QprojParams& pg, const KvAppendParams& pm, cudaStream_t stream);
cudaError_t launch_out_proj(const CUtensorMap& tw, const CUtensorMap& ta, const QprojParams& pg,
                            __nv_bfloat16* y, int64_t y_stride, cudaStream_t stream);
cudaError_t launch_lse_merge(const LseMergeParams& p, cudaStream_t stream);
}  // namespace mfa

using namespace mfa;

namespace {

thread_local cudaError_t t_last_cuda_error = cudaSuccess;

// Records a failed CUDA call for mfa_last_cuda_error_string(); returns MFA_ERR_CUDA.
int cuda_fail(cudaError_t e) {
  t_last_cuda_error = e;
  return MFA_ERR_CUDA;
}

constexpr int kMaxDevices = 64;

// ---------------------------------------------------------------------------
// device facts and the driver's tensor-map encoder
// ---------------------------------------------------------------------------
struct DeviceInfo {
  bool ok = false;
  int sms = 0;
  int cc_major = 0, cc_minor = 0;
};

std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int current_device(DeviceInfo* info) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MFA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ok) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MFA_ERR_CUDA;
    d.sms = prop.multiProcessorCount;
    d.cc_major = prop.major;
    d.cc_minor = prop.minor;
    d.ok = true;
  }
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
      return MFA_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  *info = d;
  if (d.cc_major != 10 || d.cc_minor != 0) return MFA_ERR_UNSUPPORTED;
  return MFA_OK;
}

// ---------------------------------------------------------------------------
// descriptor checks
// ---------------------------------------------------------------------------
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int elem_size(int dtype) {
  switch (dtype) {
    case MFA_BF16: return 2;
    case MFA_F32: return 4;
    case MFA_FP8_E4M3: return 1;
    case MFA_I32: return 4;
    default: return 0;
  }
}

bool well_formed(const mfa_tensor* t, int ndim) {
  if (!t || !t->data || t->ndim != ndim || elem_size(t->dtype) == 0) return false;
  for (int i = 0; i < ndim; ++i)
    if (t->shape[i] < 0 || t->stride[i] < 0) return false;
  return true;
}

CUresult encode_3d(CUtensorMap* map, CUtensorMapDataType type, int esize, const void* base,
                   uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1_elems, uint64_t s2_elems,
                   uint32_t b0, uint32_t b1) {
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1_elems * esize, s2_elems * esize};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(map, type, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Cache [B][L][256] (or page pool [P][page_size][256]) with each 512-byte
// (bf16) or 256-byte (E4M3) token row viewed as 128-byte chunks placed after
// the token dimension: {chunk elements, tokens, chunks, B or P} (strides:
// token, 128 B, sequence or page). One box of {chunk, 128, 2, 1} lands as two
// 128-row regions of 16 KB: for bf16 one item (head dims 0-127 or 128-255),
// for E4M3 the whole tensor tile.
CUresult encode_kv_chunked(CUtensorMap* map, CUtensorMapDataType type, int esize,
                           const void* base, uint64_t tokens, uint64_t batch,
                           uint64_t token_stride_elems, uint64_t batch_stride_elems) {
  const cuuint64_t inner = 128 / esize;
  const cuuint64_t dims[4] = {inner, tokens, kDim / inner, batch};
  const cuuint64_t strides[3] = {token_stride_elems * esize, 128, batch_stride_elems * esize};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(inner), 128, 2, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return g_encode(map, type, 4, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

CUresult encode_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
                   uint64_t row_stride_elems, uint32_t b0, uint32_t b1) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {row_stride_elems * 2};
  const cuuint32_t box[2] = {b0, b1};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// Row-major weight [K][N] viewed as {64 features, K, N / 64 feature chunks}
// (strides: row, 128 B): one box of {64, 64, 2} is a 128-feature x 64-k tile,
// landing as its two 64-feature halves 8 KB apart (one TMA op per stage).
CUresult encode_w3d(CUtensorMap* map, const void* base, uint64_t n, uint64_t k,
                    uint64_t row_stride_elems) {
  const cuuint64_t dims[3] = {64, k, n / 64};
  const cuuint64_t strides[2] = {row_stride_elems * 2, 128};
  const cuuint32_t box[3] = {64, 64, 2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

// ---------------------------------------------------------------------------
// per-device cached workspaces of the plain entry points
// ---------------------------------------------------------------------------
struct CachedWs {
  void* ptr = nullptr;
  size_t bytes = 0;
};
CachedWs g_ws_decode[kMaxDevices], g_ws_qproj[kMaxDevices];

int cached_workspace(CachedWs* table, size_t need, bool zero, void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MFA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  CachedWs& w = table[dev];
  if (w.bytes < need) {
    if (w.ptr) {
      cudaDeviceSynchronize();
      cudaFree(w.ptr);
      w.ptr = nullptr;
      w.bytes = 0;
    }
    void* p = nullptr;
    if (cudaMalloc(&p, need) != cudaSuccess) return MFA_ERR_CUDA;
    if (zero && cudaMemset(p, 0, need) != cudaSuccess) {
      cudaFree(p);
      return MFA_ERR_CUDA;
    }
    w.ptr = p;
    w.bytes = need;
  }
  *out = w.ptr;
  return MFA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Decode workspace: the hand-off words between the attention and the combine
// kernel (per-sequence plan words, per-slot flags), then the partial outputs of
// split sequences, their log-sum-exp values and the L2 warm-up hint. Every
// word the combine kernel reads is written in the same call before it may
// start, so the workspace needs no initialisation and keeps nothing between
// calls that a later call relies on.
struct DecodeWsLayout {
  size_t plan_off, flag_off, o_off, lse_off, hint_off, total;
  int slots;
};

DecodeWsLayout decode_ws_layout(int batch, int num_splits, int grid) {
  DecodeWsLayout l;
  const size_t B = static_cast<size_t>(batch);
  l.slots = num_splits == 0 ? 2 * grid : batch * num_splits;
  l.plan_off = 0;
  l.flag_off = align256(B * sizeof(unsigned long long));
  l.o_off = align256(l.flag_off + static_cast<size_t>(l.slots) * sizeof(unsigned));
  l.lse_off = align256(l.o_off + static_cast<size_t>(l.slots) * kPartialFloats * sizeof(float));
  l.hint_off = align256(l.lse_off + static_cast<size_t>(l.slots) * kHeads * sizeof(float));
  l.total = align256(l.hint_off + static_cast<size_t>(grid) * 2 * sizeof(int));
  return l;
}

// Limit of the combine kernel's waits for partials (the attention kernel's own
// waits have the same 2 s limit, fixed).
constexpr unsigned long long kDecodeWaitNs = 2000000000ull;

constexpr int kMaxSplits = 1024;

int decode_grid(const DeviceInfo& d, int batch, int num_splits) {
  if (num_splits == 0) return d.sms;
  const long long units = static_cast<long long>(batch) * num_splits;
  return static_cast<int>(units < d.sms ? units : d.sms);
}

// ---------------------------------------------------------------------------
// query projection workspace: fp32 partials, counters, interleaved latent
// ---------------------------------------------------------------------------
struct QprojWsLayout {
  size_t part_off, cnt_off, lat_off, total;
  int splits;
};

// The split-K counters sit in a fixed region at the start of the workspace so
// that calls of any shape reuse the same zero-filled counters (every call
// leaves them zero); partials and the latent follow.
constexpr int kMaxCounters = 1024;  // output tiles of the first GEMM: rank <= 128 * 1024

QprojWsLayout qproj_ws_layout(int batch, int dm, int rank, int sms) {
  QprojWsLayout l;
  const int k_blocks = dm / 64;
  const int m_tiles = rank / 128;
  int splits = m_tiles > 0 ? sms / m_tiles : 1;
  if (splits < 1) splits = 1;
  if (splits > k_blocks) splits = k_blocks;
  l.splits = splits;
  l.cnt_off = 0;
  l.part_off = align256(static_cast<size_t>(kMaxCounters) * sizeof(int));
  l.lat_off = align256(l.part_off + static_cast<size_t>(splits) * batch * rank * sizeof(float));
  l.total = align256(l.lat_off + static_cast<size_t>(2 * batch) * rank * 2);
  return l;
}

}  // namespace

// ===========================================================================
// public entry points
// ===========================================================================
extern "C" {

const char* mfa_error_string(int code) {
  switch (code) {
    case MFA_OK: return "MFA_OK";
    case MFA_ERR_INVALID_ARG: return "MFA_ERR_INVALID_ARG: invalid argument";
    case MFA_ERR_UNSUPPORTED: return "MFA_ERR_UNSUPPORTED: unsupported shape, dtype or device";
    case MFA_ERR_CUDA: return "MFA_ERR_CUDA: CUDA call or kernel launch failed";
    case MFA_ERR_WORKSPACE: return "MFA_ERR_WORKSPACE: workspace missing or too small";
    case MFA_ERR_BAD_INDEX: return "MFA_ERR_BAD_INDEX: page id or sequence length out of range";
    case MFA_ERR_TIMEOUT: return "MFA_ERR_TIMEOUT: an in-kernel wait exceeded its time limit";
    default: return "unknown mfa status code";
  }
}

int mfa_version(void) { return 100; }

#ifdef MFA_TRACE
// Trace builds only: copy the pipeline trace (see decode_kernel.cu) to host memory.
int mfa_debug_read_trace(void* dst, size_t bytes) {
  if (bytes > sizeof(g_mfa_trace)) bytes = sizeof(g_mfa_trace);
  return cudaMemcpyFromSymbol(dst, g_mfa_trace, bytes) == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
}
int mfa_debug_read_timeline(void* dst, size_t bytes) {
  if (bytes > sizeof(g_mfa_gt)) bytes = sizeof(g_mfa_gt);
  return cudaMemcpyFromSymbol(dst, g_mfa_gt, bytes) == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
}
int mfa_debug_reset_timeline(void) {
  static int zeros[2 * kGtCtas] = {0};
  return cudaMemcpyToSymbol(g_mfa_cnt, zeros, sizeof zeros) == cudaSuccess ? MFA_OK : MFA_ERR_CUDA;
}
#endif

const char* mfa_last_cuda_error_string(void) {
  return t_last_cuda_error == cudaSuccess ? "no CUDA error recorded"
                                          : cudaGetErrorString(t_last_cuda_error);
}

size_t mfa_decode_workspace_size(int batch, int num_splits) {
  if (batch <= 0 || num_splits < 0 || num_splits > kMaxSplits) return 0;
  DeviceInfo d;
  const int rc = current_device(&d);
  if (rc != MFA_OK && rc != MFA_ERR_UNSUPPORTED) return 0;
  return decode_ws_layout(batch, num_splits, decode_grid(d, batch, num_splits)).total;
}

}  // extern "C"

namespace {

// A 4-D grouped-query cache [*, tokens, 2, 128] as the 3-D view [*, tokens, 256]
// the kernels read (a token's two group rows must be adjacent: stride 128).
bool gqa_cache_view(const mfa_tensor* t, mfa_tensor* view) {
  if (!well_formed(t, 4) || t->shape[2] != 2 || t->shape[3] != kDim / 2 ||
      t->stride[3] != 1 || t->stride[2] != kDim / 2)
    return false;
  *view = *t;
  view->ndim = 3;
  view->shape[2] = kDim;
  view->stride[2] = 1;
  view->shape[3] = 0;
  view->stride[3] = 0;
  return true;
}

// Validates every argument (host only, no CUDA call) and, unless
// validate_only, encodes the tensor maps and launches.
int decode_impl(const mfa_tensor* q, const mfa_tensor* k_cache, const mfa_tensor* v_cache,
                const mfa_tensor* page_table, const mfa_tensor* seq_lens, mfa_tensor* out,
                float softmax_scale, int kv_dtype, float k_scale, float v_scale, int num_splits,
                mfa_tensor* lse_out, void* workspace, size_t workspace_bytes, mfa_stream_t stream,
                bool validate_only, bool gqa = false, bool q_after_proj = false) {
  // ---- shapes and dtypes ----
  // grouped-query mode: q and out [B, 64, 128], caches [*, tokens, 2, 128] bf16,
  // viewed as [*, tokens, 256]
  mfa_tensor kview, vview;
  if (gqa) {
    if (!gqa_cache_view(k_cache, &kview) || !gqa_cache_view(v_cache, &vview))
      return well_formed(k_cache, 4) && well_formed(v_cache, 4) ? MFA_ERR_UNSUPPORTED
                                                                : MFA_ERR_INVALID_ARG;
    if (kv_dtype != MFA_BF16) return MFA_ERR_UNSUPPORTED;
    k_cache = &kview;
    v_cache = &vview;
  }
  const int qdim = gqa ? kDim / 2 : kDim;
  if (!well_formed(q, 3) || !well_formed(k_cache, 3) || !well_formed(v_cache, 3) ||
      !well_formed(seq_lens, 1) || !well_formed(out, 3))
    return MFA_ERR_INVALID_ARG;
  if (!(softmax_scale == softmax_scale) || !(k_scale == k_scale) || !(v_scale == v_scale))
    return MFA_ERR_INVALID_ARG;
  if (num_splits < 0 || num_splits > kMaxSplits) return MFA_ERR_INVALID_ARG;
  const int64_t B = q->shape[0];
  if (B <= 0 || B > (1 << 20)) return MFA_ERR_INVALID_ARG;
  if (q->dtype != MFA_BF16) return MFA_ERR_INVALID_ARG;
  if (q->shape[1] != kHeads || q->shape[2] != qdim) return MFA_ERR_UNSUPPORTED;
  if (q->stride[2] != 1 || q->stride[1] % 8 || q->stride[0] % 8) return MFA_ERR_INVALID_ARG;
  if (kv_dtype != MFA_BF16 && kv_dtype != MFA_FP8_E4M3) return MFA_ERR_INVALID_ARG;
  if (k_cache->dtype != kv_dtype || v_cache->dtype != kv_dtype) return MFA_ERR_INVALID_ARG;
  if (kv_dtype == MFA_BF16 && (k_scale != 1.f || v_scale != 1.f)) return MFA_ERR_INVALID_ARG;
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || k_scale > 1e30f || v_scale > 1e30f)
    return MFA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (k_cache->shape[i] != v_cache->shape[i]) return MFA_ERR_INVALID_ARG;
  if (k_cache->shape[2] != kDim) return MFA_ERR_UNSUPPORTED;
  const int esz = elem_size(kv_dtype);
  for (const mfa_tensor* t : {k_cache, v_cache}) {
    if (t->stride[2] != 1 || (t->stride[1] * esz) % 16 || (t->stride[0] * esz) % 16 ||
        !aligned16(t->data))
      return MFA_ERR_INVALID_ARG;
  }
  if (!aligned16(q->data)) return MFA_ERR_INVALID_ARG;
  if (seq_lens->dtype != MFA_I32 || seq_lens->shape[0] != B || seq_lens->stride[0] != 1)
    return MFA_ERR_INVALID_ARG;
  if (out->dtype != MFA_BF16 && out->dtype != MFA_F32) return MFA_ERR_INVALID_ARG;
  if (out->shape[0] != B || out->shape[1] != kHeads || out->shape[2] != qdim ||
      out->stride[2] != 1)
    return MFA_ERR_INVALID_ARG;
  if (lse_out) {
    if (!well_formed(lse_out, 2) || lse_out->dtype != MFA_F32 || lse_out->shape[0] != B ||
        lse_out->shape[1] != kHeads || lse_out->stride[1] != 1)
      return MFA_ERR_INVALID_ARG;
  }
  const bool paged = page_table != nullptr;
  int page_size = 0, max_pages = 0, num_pages = 0;
  int64_t cap = 0;
  if (paged) {
    if (!well_formed(page_table, 2) || page_table->dtype != MFA_I32 ||
        page_table->shape[0] != B || page_table->stride[1] != 1)
      return MFA_ERR_INVALID_ARG;
    page_size = static_cast<int>(k_cache->shape[1]);
    if (page_size != 16 && page_size != 32 && page_size != 64 && page_size != 128 &&
        page_size != 256)
      return MFA_ERR_UNSUPPORTED;
    if (k_cache->shape[0] <= 0 || k_cache->shape[0] > (1ll << 31) - 1) return MFA_ERR_INVALID_ARG;
    num_pages = static_cast<int>(k_cache->shape[0]);
    if (page_table->shape[1] <= 0 || page_table->shape[1] > (1 << 24)) return MFA_ERR_INVALID_ARG;
    max_pages = static_cast<int>(page_table->shape[1]);
    cap = static_cast<int64_t>(max_pages) * page_size;
    if (k_cache->stride[1] != kDim || v_cache->stride[1] != kDim) return MFA_ERR_INVALID_ARG;
  } else {
    if (k_cache->shape[0] != B) return MFA_ERR_INVALID_ARG;
    cap = k_cache->shape[1];
  }
  if (cap > (1 << 30)) return MFA_ERR_UNSUPPORTED;
  if (validate_only) return MFA_OK;

  DeviceInfo dev;
  int rc = current_device(&dev);
  if (rc != MFA_OK) return rc;
  const int grid = decode_grid(dev, static_cast<int>(B), num_splits);
  const DecodeWsLayout wl = decode_ws_layout(static_cast<int>(B), num_splits, grid);
  if (!workspace || workspace_bytes < wl.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return MFA_ERR_WORKSPACE;

  // ---- tensor maps ----
  CUtensorMap tq, tk, tv;
  // q boxes of 64 dims x 64 heads (grouped-query mode: x 32 heads, one group)
  if (encode_3d(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, q->data, qdim, kHeads, B, q->stride[1],
                q->stride[0], 64, gqa ? kHeads / 2 : kHeads) != CUDA_SUCCESS)
    return MFA_ERR_INVALID_ARG;
  const int rows = paged ? (page_size < kTile ? page_size : kTile) : kTile;
  const uint64_t d1 = paged ? static_cast<uint64_t>(page_size) : static_cast<uint64_t>(cap);
  const uint64_t d2 = paged ? static_cast<uint64_t>(num_pages) : static_cast<uint64_t>(B);
  if (cap == 0 && !paged) {
    // a zero-length cache: nothing is ever loaded, but a map needs extent >= 1
  }
  const uint64_t d1s = d1 > 0 ? d1 : 1;
  // bf16: boxes of 64 dims (128 bytes); E4M3: boxes of 128 dims (128 bytes)
  const bool fp8 = kv_dtype == MFA_FP8_E4M3;
  const CUtensorMapDataType kv_type =
      fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint32_t box0 = fp8 ? 128 : 64;
  if (rows == kTile) {
    // contiguous, or pages of >= 128 tokens: tokens = cap or page_size, outer
    // index = sequence or page
    if (encode_kv_chunked(&tk, kv_type, esz, k_cache->data, d1s, d2, k_cache->stride[1],
                          k_cache->stride[0]) != CUDA_SUCCESS ||
        encode_kv_chunked(&tv, kv_type, esz, v_cache->data, d1s, d2, v_cache->stride[1],
                          v_cache->stride[0]) != CUDA_SUCCESS)
      return MFA_ERR_INVALID_ARG;
  } else if (encode_3d(&tk, kv_type, esz, k_cache->data, kDim, d1s, d2, k_cache->stride[1],
                       k_cache->stride[0], box0, rows) != CUDA_SUCCESS ||
             encode_3d(&tv, kv_type, esz, v_cache->data, kDim, d1s, d2, v_cache->stride[1],
                       v_cache->stride[0], box0, rows) != CUDA_SUCCESS) {
    return MFA_ERR_INVALID_ARG;
  }

  DecodeParams p;
  std::memset(&p, 0, sizeof p);
  p.seq_lens = static_cast<const int*>(seq_lens->data);
  p.batch = static_cast<int>(B);
  p.cap_tokens = static_cast<int>(cap);
  p.paged = paged;
  p.page_size = page_size;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.page_table = paged ? static_cast<const int*>(page_table->data) : nullptr;
  p.pt_stride = paged ? page_table->stride[0] : 0;
  p.num_splits = num_splits;
  p.grid = grid;
  p.score_log2 = softmax_scale * k_scale * 1.4426950408889634f;
  p.out_scale = v_scale;
  p.out = out->data;
  p.out_f32 = out->dtype == MFA_F32;
  p.out_sb = out->stride[0];
  p.out_sh = out->stride[1];
  p.lse_out = lse_out ? static_cast<float*>(lse_out->data) : nullptr;
  p.lse_sb = lse_out ? lse_out->stride[0] : 0;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.ws_o = reinterpret_cast<float*>(ws + wl.o_off);
  p.ws_lse = reinterpret_cast<float*>(ws + wl.lse_off);
  p.ws_hint = reinterpret_cast<int*>(ws + wl.hint_off);
  p.ws_plan = reinterpret_cast<unsigned long long*>(ws + wl.plan_off);
  p.ws_flag = reinterpret_cast<unsigned*>(ws + wl.flag_off);
  p.wait_ns = kDecodeWaitNs;
  p.gqa = gqa ? 1 : 0;
  p.q_after_proj = q_after_proj ? 1 : 0;
  const cudaError_t err =
      launch_decode(paged, fp8, tq, tk, tv, p, reinterpret_cast<cudaStream_t>(stream));
  return err == cudaSuccess ? MFA_OK : cuda_fail(err);
}

}  // namespace

extern "C" {

int mfa_decode_attention_ex(const mfa_tensor* q, const mfa_tensor* k_cache,
                            const mfa_tensor* v_cache, const mfa_tensor* page_table,
                            const mfa_tensor* seq_lens, mfa_tensor* out, float softmax_scale,
                            int kv_dtype, float k_scale, float v_scale, int num_splits,
                            mfa_tensor* lse_out, void* workspace, size_t workspace_bytes,
                            mfa_stream_t stream) {
  return decode_impl(q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale, kv_dtype,
                     k_scale, v_scale, num_splits, lse_out, workspace, workspace_bytes, stream,
                     false);
}

int mfa_gqa_decode_attention(const mfa_tensor* q, const mfa_tensor* k_cache,
                             const mfa_tensor* v_cache, const mfa_tensor* page_table,
                             const mfa_tensor* seq_lens, mfa_tensor* out, float softmax_scale,
                             int num_splits, mfa_tensor* lse_out, void* workspace,
                             size_t workspace_bytes, mfa_stream_t stream) {
  return decode_impl(q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale, MFA_BF16, 1.f,
                     1.f, num_splits, lse_out, workspace, workspace_bytes, stream, false, true);
}

int mfa_decode_attention(const mfa_tensor* q, const mfa_tensor* k_cache,
                         const mfa_tensor* v_cache, const mfa_tensor* page_table,
                         const mfa_tensor* seq_lens, mfa_tensor* out, float softmax_scale,
                         int kv_dtype, mfa_stream_t stream) {
  const int vrc = decode_impl(q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale,
                              kv_dtype, 1.f, 1.f, 0, nullptr, nullptr, 0, stream, true);
  if (vrc != MFA_OK) return vrc;
  const size_t need = mfa_decode_workspace_size(static_cast<int>(q->shape[0]), 0);
  if (need == 0) return MFA_ERR_CUDA;
  void* ws = nullptr;
  const int rc = cached_workspace(g_ws_decode, need, false, &ws);
  if (rc != MFA_OK) return rc;
  return mfa_decode_attention_ex(q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale,
                                 kv_dtype, 1.f, 1.f, 0, nullptr, ws, need, stream);
}

size_t mfa_query_proj_workspace_size(int batch, int dm, int rank) {
  if (batch <= 0 || dm <= 0 || rank <= 0) return 0;
  DeviceInfo d;
  const int rc = current_device(&d);
  if (rc != MFA_OK && rc != MFA_ERR_UNSUPPORTED) return 0;
  return qproj_ws_layout(batch, dm, rank, d.sms).total;
}

}  // extern "C"

namespace {

int qproj_impl(const mfa_tensor* x, const mfa_tensor* w_qa, const mfa_tensor* w_qb,
               mfa_tensor* q_out, void* workspace, size_t workspace_bytes, mfa_stream_t stream,
               bool validate_only) {
  if (!well_formed(x, 2) || !well_formed(w_qa, 2) || !well_formed(w_qb, 2) ||
      !well_formed(q_out, 2))
    return MFA_ERR_INVALID_ARG;
  for (const mfa_tensor* t : std::initializer_list<const mfa_tensor*>{x, w_qa, w_qb, q_out})
    if (t->dtype != MFA_BF16 || t->stride[1] != 1 || t->stride[0] % 8 || !aligned16(t->data))
      return MFA_ERR_INVALID_ARG;
  const int64_t B = x->shape[0], Dm = x->shape[1], R = w_qa->shape[1], N = w_qb->shape[1];
  if (w_qa->shape[0] != Dm || w_qb->shape[0] != R || q_out->shape[0] != B || q_out->shape[1] != N)
    return MFA_ERR_INVALID_ARG;
  if (B < 1 || B > 128 || Dm % 64 || R % 128 || N % 128 || Dm <= 0 || R <= 0 || N <= 0 ||
      Dm > (1 << 20) || R > 128 * kMaxCounters || N > (1 << 24))
    return MFA_ERR_UNSUPPORTED;
  if (validate_only) return MFA_OK;

  DeviceInfo dev;
  int rc = current_device(&dev);
  if (rc != MFA_OK) return rc;
  const QprojWsLayout wl = qproj_ws_layout(static_cast<int>(B), static_cast<int>(Dm),
                                           static_cast<int>(R), dev.sms);
  if (!workspace || workspace_bytes < wl.total || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return MFA_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  __nv_bfloat16* latent = reinterpret_cast<__nv_bfloat16*>(ws + wl.lat_off);

  const int n1 = static_cast<int>((B + 15) / 16 * 16);
  const int n2 = static_cast<int>((2 * B + 15) / 16 * 16);
  CUtensorMap tw1, tx, tw2, tl;
  if (encode_2d(&tw1, w_qa->data, R, Dm, w_qa->stride[0], 64, 64) != CUDA_SUCCESS ||
      encode_2d(&tx, x->data, Dm, B, x->stride[0], 64, n1) != CUDA_SUCCESS ||
      encode_2d(&tw2, w_qb->data, N, R, w_qb->stride[0], 64, 64) != CUDA_SUCCESS ||
      encode_2d(&tl, latent, R, 2 * B, R, 64, n2) != CUDA_SUCCESS)
    return MFA_ERR_INVALID_ARG;

  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int m1 = static_cast<int>(R / 128), m2 = static_cast<int>(N / 128);
  if (B <= 8 && m1 < kQprojDone && m1 * wl.splits <= dev.sms && m2 <= dev.sms &&
      qproj_fused_fits(n1, n2, static_cast<int>(R / 64))) {
    // both GEMMs in one persistent kernel (see qproj_kernel.cu)
    QprojFusedParams pf;
    std::memset(&pf, 0, sizeof pf);
    pf.batch = static_cast<int>(B);
    pf.k1_blocks = static_cast<int>(Dm / 64);
    pf.k2_blocks = static_cast<int>(R / 64);
    pf.m1_tiles = m1;
    pf.m2_tiles = m2;
    pf.splits = wl.splits;
    pf.n1 = n1;
    pf.n2 = n2;
    pf.rank = static_cast<int>(R);
    pf.partials = reinterpret_cast<float*>(ws + wl.part_off);
    pf.counters = reinterpret_cast<int*>(ws + wl.cnt_off);
    pf.latent = latent;
    pf.q_out = static_cast<__nv_bfloat16*>(q_out->data);
    pf.q_stride = q_out->stride[0];
    CUtensorMap tw1v, tw2v;
    if (encode_w3d(&tw1v, w_qa->data, R, Dm, w_qa->stride[0]) != CUDA_SUCCESS ||
        encode_w3d(&tw2v, w_qb->data, N, R, w_qb->stride[0]) != CUDA_SUCCESS)
      return MFA_ERR_INVALID_ARG;
    const int grid = m1 * wl.splits > m2 ? m1 * wl.splits : m2;
    const cudaError_t ef = launch_qproj_fused(tw1v, tx, tw2v, tl, pf, grid, st);
    return ef == cudaSuccess ? MFA_OK : cuda_fail(ef);
  }

  QprojParams p1;
  std::memset(&p1, 0, sizeof p1);
  p1.batch = static_cast<int>(B);
  p1.k_blocks = static_cast<int>(Dm / 64);
  p1.m_total = static_cast<int>(R);
  p1.splits = wl.splits;
  p1.n_cols = n1;
  p1.mode = 0;
  p1.partials = reinterpret_cast<float*>(ws + wl.part_off);
  p1.counters = reinterpret_cast<int*>(ws + wl.cnt_off);
  p1.latent = latent;
  cudaError_t e = launch_qproj(tw1, tx, p1, static_cast<int>(R / 128), st);
  if (e != cudaSuccess) return cuda_fail(e);

  QprojParams p2 = p1;
  p2.k_blocks = static_cast<int>(R / 64);
  p2.m_total = static_cast<int>(N);
  p2.splits = 1;
  p2.n_cols = n2;
  p2.mode = 1;
  p2.q_out = static_cast<__nv_bfloat16*>(q_out->data);
  p2.q_stride = q_out->stride[0];
  e = launch_qproj(tw2, tl, p2, static_cast<int>(N / 128), st);
  if (e != cudaSuccess) return cuda_fail(e);
  return MFA_OK;
}

}  // namespace

extern "C" {

int mfa_query_proj_ex(const mfa_tensor* x, const mfa_tensor* w_qa, const mfa_tensor* w_qb,
                      mfa_tensor* q_out, void* workspace, size_t workspace_bytes,
                      mfa_stream_t stream) {
  return qproj_impl(x, w_qa, w_qb, q_out, workspace, workspace_bytes, stream, false);
}

size_t mfa_qproj_decode_workspace_size(int batch, int dm, int rank, int num_splits) {
  const size_t a = mfa_query_proj_workspace_size(batch, dm, rank);
  const size_t b = mfa_decode_workspace_size(batch, num_splits);
  return a == 0 || b == 0 ? 0 : align256(a) + b;
}

int mfa_qproj_decode_attention(const mfa_tensor* x, const mfa_tensor* w_qa,
                               const mfa_tensor* w_qb, mfa_tensor* q_out,
                               const mfa_tensor* k_cache, const mfa_tensor* v_cache,
                               const mfa_tensor* page_table, const mfa_tensor* seq_lens,
                               mfa_tensor* out, float softmax_scale, int kv_dtype, float k_scale,
                               float v_scale, int num_splits, mfa_tensor* lse_out,
                               void* workspace, size_t workspace_bytes, mfa_stream_t stream) {
  // q_out [B, 64 * 256] is the attention's q [B, 64, 256]
  if (!well_formed(q_out, 2) || q_out->shape[1] != static_cast<int64_t>(kHeads) * kDim ||
      q_out->stride[1] != 1 || !well_formed(x, 2) || !well_formed(w_qa, 2))
    return MFA_ERR_INVALID_ARG;
  mfa_tensor q3 = *q_out;
  q3.ndim = 3;
  q3.shape[1] = kHeads;
  q3.shape[2] = kDim;
  q3.stride[1] = kDim;
  q3.stride[2] = 1;
  // validate both halves before launching either
  int rc = qproj_impl(x, w_qa, w_qb, q_out, nullptr, 0, stream, true);
  if (rc != MFA_OK) return rc;
  rc = decode_impl(&q3, k_cache, v_cache, page_table, seq_lens, out, softmax_scale, kv_dtype,
                   k_scale, v_scale, num_splits, lse_out, nullptr, 0, stream, true);
  if (rc != MFA_OK) return rc;
  const size_t qbytes = mfa_query_proj_workspace_size(static_cast<int>(x->shape[0]),
                                                      static_cast<int>(x->shape[1]),
                                                      static_cast<int>(w_qa->shape[1]));
  const size_t dbytes = mfa_decode_workspace_size(static_cast<int>(x->shape[0]), num_splits);
  if (qbytes == 0 || dbytes == 0) return MFA_ERR_CUDA;
  const size_t split = align256(qbytes);
  if (!workspace || workspace_bytes < split + dbytes) return MFA_ERR_WORKSPACE;
  rc = qproj_impl(x, w_qa, w_qb, q_out, workspace, qbytes, stream, false);
  if (rc != MFA_OK) return rc;
  // launched with programmatic dependent launch as the projection's CTAs
  // finish: the projection let it launch only after its own dependency wait,
  // so the attention plans and streams K/V at once and waits for the
  // projection grid only before it reads q
  return decode_impl(&q3, k_cache, v_cache, page_table, seq_lens, out, softmax_scale, kv_dtype,
                     k_scale, v_scale, num_splits, lse_out, static_cast<uint8_t*>(workspace) + split,
                     workspace_bytes - split, stream, false, false, true);
}

int mfa_query_proj(const mfa_tensor* x, const mfa_tensor* w_qa, const mfa_tensor* w_qb,
                   mfa_tensor* q_out, mfa_stream_t stream) {
  const int vrc = qproj_impl(x, w_qa, w_qb, q_out, nullptr, 0, stream, true);
  if (vrc != MFA_OK) return vrc;
  const size_t need = mfa_query_proj_workspace_size(static_cast<int>(x->shape[0]),
                                                    static_cast<int>(x->shape[1]),
                                                    static_cast<int>(w_qa->shape[1]));
  if (need == 0) return MFA_ERR_CUDA;
  void* ws = nullptr;
  const int rc = cached_workspace(g_ws_qproj, need, true, &ws);
  if (rc != MFA_OK) return rc;
  return mfa_query_proj_ex(x, w_qa, w_qb, q_out, ws, need, stream);
}

int mfa_read_status(mfa_stream_t stream, int reset, int* status_out) {
  if (!status_out) return MFA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  e = cudaMemcpyFromSymbol(&v, g_mfa_status, sizeof v);
  if (e != cudaSuccess) return cuda_fail(e);
  if (reset) {
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_mfa_status, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  *status_out = v;
  return MFA_OK;
}

}  // extern "C"

// ===========================================================================
// Allocation-free decode attention: the split workspace lives in a fixed
// device array owned by the library instead of memory the caller or the
// library allocates per call.
// ===========================================================================
static constexpr size_t kNoAllocScratchBytes = static_cast<size_t>(24) << 20;  // 24 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// Device address of g_noalloc_scratch on each device, looked up on the first
// call made with that device current (the host-side symbol is only a handle).
void* g_noalloc_addr[kMaxDevices] = {};
}  // namespace

extern "C" int mfa_decode_attention_noalloc(const mfa_tensor* q, const mfa_tensor* k_cache,
                                            const mfa_tensor* v_cache, const mfa_tensor* page_table,
                                            const mfa_tensor* seq_lens, mfa_tensor* out,
                                            float softmax_scale, int kv_dtype, float k_scale,
                                            float v_scale, int num_splits, mfa_tensor* lse_out,
                                            mfa_stream_t stream) {
  const int vrc = decode_impl(q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale,
                              kv_dtype, k_scale, v_scale, num_splits, lse_out, nullptr, 0, stream,
                              true);
  if (vrc != MFA_OK) return vrc;
  const size_t need = mfa_decode_workspace_size(static_cast<int>(q->shape[0]), num_splits);
  if (need == 0) return MFA_ERR_CUDA;
  if (need > kNoAllocScratchBytes) return MFA_ERR_WORKSPACE;  // batch x splits too large
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return MFA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_noalloc_addr[dev]) {
      e = cudaGetSymbolAddress(&g_noalloc_addr[dev], g_noalloc_scratch);
      if (e != cudaSuccess) {
        g_noalloc_addr[dev] = nullptr;
        return cuda_fail(e);
      }
    }
    scratch = g_noalloc_addr[dev];
  }
  return decode_impl(q, k_cache, v_cache, page_table, seq_lens, out, softmax_scale, kv_dtype,
                     k_scale, v_scale, num_splits, lse_out, scratch, kNoAllocScratchBytes, stream,
                     false);
}

// ===========================================================================
// Failure-path self-test: the combine kernel waits for two partials that no
// attention kernel publishes (their flags stay zero: nothing writes them), so
// its bounded waits run out and it records MFA_ERR_TIMEOUT.
// ===========================================================================
static __device__ int g_selftest_len[1] = {2 * kTile};  // one sequence, two tiles
static __device__ unsigned g_selftest_flag[2];            // never set
static __device__ __align__(16) float g_selftest_out[kHeads * kDim];

namespace {
struct SelftestAddr {
  void* len = nullptr;
  void* flag = nullptr;
  void* out = nullptr;
};
SelftestAddr g_selftest_addr[kMaxDevices];
}  // namespace

extern "C" int mfa_selftest_wait_timeout(unsigned long long wait_ns, mfa_stream_t stream) {
  if (wait_ns < 1 || wait_ns > 10000000000ull) return MFA_ERR_INVALID_ARG;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return MFA_ERR_UNSUPPORTED;
  SelftestAddr a;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    SelftestAddr& s = g_selftest_addr[dev];
    if (!s.len) {
      if ((e = cudaGetSymbolAddress(&s.flag, g_selftest_flag)) != cudaSuccess ||
          (e = cudaGetSymbolAddress(&s.out, g_selftest_out)) != cudaSuccess ||
          (e = cudaGetSymbolAddress(&s.len, g_selftest_len)) != cudaSuccess) {
        s = SelftestAddr{};
        return cuda_fail(e);
      }
    }
    a = s;
  }
  DecodeParams p;
  std::memset(&p, 0, sizeof p);
  p.seq_lens = static_cast<const int*>(a.len);
  p.batch = 1;
  p.cap_tokens = 2 * kTile;
  p.num_splits = 2;  // tiles [0, 1) and [1, 2): partial slots 0 and 1
  p.grid = 2;
  p.out = a.out;
  p.out_f32 = 1;
  p.out_sb = static_cast<int64_t>(kHeads) * kDim;
  p.out_sh = kDim;
  p.ws_o = static_cast<float*>(a.out);  // never read: the merge is skipped
  p.ws_lse = static_cast<float*>(a.out);
  p.ws_flag = static_cast<unsigned*>(a.flag);
  p.wait_ns = wait_ns;
  e = launch_combine_only(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MFA_OK : cuda_fail(e);
}

// ===========================================================================
// New-token key/value projection and cache append
// ===========================================================================
namespace {

// Split-K factor of the append projection: the four 128-feature tiles of
// [W_k | W_v] times this many k-ranges fill the SMs.
int kv_append_splits(int64_t hidden, int sms) {
  int s = sms / 4;
  if (s < 1) s = 1;
  if (s > hidden / 64) s = static_cast<int>(hidden / 64);
  return s;
}

size_t kv_append_ws_bytes(int64_t batch, int64_t hidden, int sms) {
  return align256(static_cast<size_t>(kv_append_splits(hidden, sms)) * batch * 2 * kDim *
                  sizeof(float));
}

}  // namespace

extern "C" {

size_t mfa_kv_append_workspace_size(int batch, int hidden) {
  if (batch <= 0 || hidden <= 0 || hidden % 64) return 0;
  DeviceInfo d;
  const int rc = current_device(&d);
  if (rc != MFA_OK && rc != MFA_ERR_UNSUPPORTED) return 0;
  return kv_append_ws_bytes(batch, hidden, d.sms);
}

int mfa_kv_append(const mfa_tensor* x, const mfa_tensor* w_k, const mfa_tensor* w_v,
                  mfa_tensor* k_cache, mfa_tensor* v_cache, const mfa_tensor* page_table,
                  const mfa_tensor* positions, int kv_dtype, float k_scale, float v_scale,
                  void* workspace, size_t workspace_bytes, mfa_stream_t stream) {
  // ---- shapes and dtypes ----
  if (!well_formed(x, 2) || !well_formed(w_k, 2) || !well_formed(w_v, 2) ||
      !well_formed(k_cache, 3) || !well_formed(v_cache, 3) || !well_formed(positions, 1))
    return MFA_ERR_INVALID_ARG;
  for (const mfa_tensor* t : std::initializer_list<const mfa_tensor*>{x, w_k, w_v})
    if (t->dtype != MFA_BF16 || t->stride[1] != 1 || t->stride[0] % 8 || !aligned16(t->data))
      return MFA_ERR_INVALID_ARG;
  const int64_t B = x->shape[0], Dm = x->shape[1];
  if (w_k->shape[0] != Dm || w_v->shape[0] != Dm || w_k->shape[1] != kDim ||
      w_v->shape[1] != kDim)
    return MFA_ERR_INVALID_ARG;
  if (B < 1 || B > 256 || Dm <= 0 || Dm % 64 || Dm > (1 << 20)) return MFA_ERR_UNSUPPORTED;
  if (kv_dtype != MFA_BF16 && kv_dtype != MFA_FP8_E4M3) return MFA_ERR_INVALID_ARG;
  if (k_cache->dtype != kv_dtype || v_cache->dtype != kv_dtype) return MFA_ERR_INVALID_ARG;
  if (!(k_scale == k_scale) || !(v_scale == v_scale)) return MFA_ERR_INVALID_ARG;
  if (kv_dtype == MFA_BF16 && (k_scale != 1.f || v_scale != 1.f)) return MFA_ERR_INVALID_ARG;
  if (!(k_scale > 0.f) || !(v_scale > 0.f) || k_scale > 1e30f || v_scale > 1e30f)
    return MFA_ERR_INVALID_ARG;
  for (int i = 0; i < 3; ++i)
    if (k_cache->shape[i] != v_cache->shape[i] || k_cache->stride[i] != v_cache->stride[i])
      return MFA_ERR_INVALID_ARG;
  if (k_cache->shape[2] != kDim || k_cache->stride[2] != 1) return MFA_ERR_INVALID_ARG;
  if (!k_cache->data || !v_cache->data) return MFA_ERR_INVALID_ARG;
  if (positions->dtype != MFA_I32 || positions->shape[0] != B || positions->stride[0] != 1)
    return MFA_ERR_INVALID_ARG;
  const bool paged = page_table != nullptr;
  int page_size = 0, max_pages = 0, num_pages = 0;
  int64_t cap = 0;
  if (paged) {
    if (!well_formed(page_table, 2) || page_table->dtype != MFA_I32 ||
        page_table->shape[0] != B || page_table->stride[1] != 1)
      return MFA_ERR_INVALID_ARG;
    if (k_cache->shape[0] <= 0 || k_cache->shape[0] > (1ll << 31) - 1 || k_cache->shape[1] <= 0 ||
        k_cache->shape[1] > (1 << 20) || page_table->shape[1] <= 0 ||
        page_table->shape[1] > (1 << 24))
      return MFA_ERR_INVALID_ARG;
    page_size = static_cast<int>(k_cache->shape[1]);
    num_pages = static_cast<int>(k_cache->shape[0]);
    max_pages = static_cast<int>(page_table->shape[1]);
    if (static_cast<int64_t>(max_pages) * page_size > (1ll << 30)) return MFA_ERR_UNSUPPORTED;
  } else {
    if (k_cache->shape[0] != B) return MFA_ERR_INVALID_ARG;
    cap = k_cache->shape[1];
    if (cap > (1 << 30)) return MFA_ERR_UNSUPPORTED;
  }

  DeviceInfo dev;
  int rc = current_device(&dev);
  if (rc != MFA_OK) return rc;
  const int splits = kv_append_splits(Dm, dev.sms);
  if (!workspace || workspace_bytes < kv_append_ws_bytes(B, Dm, dev.sms) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return MFA_ERR_WORKSPACE;

  const int n_cols = static_cast<int>((B + 15) / 16 * 16);
  CUtensorMap twk, twv, tx;
  if (encode_2d(&twk, w_k->data, kDim, Dm, w_k->stride[0], 64, 64) != CUDA_SUCCESS ||
      encode_2d(&twv, w_v->data, kDim, Dm, w_v->stride[0], 64, 64) != CUDA_SUCCESS ||
      encode_2d(&tx, x->data, Dm, B, x->stride[0], 64, n_cols) != CUDA_SUCCESS)
    return MFA_ERR_INVALID_ARG;

  QprojParams pg;
  std::memset(&pg, 0, sizeof pg);
  pg.batch = static_cast<int>(B);
  pg.k_blocks = static_cast<int>(Dm / 64);
  pg.m_total = 2 * kDim;
  pg.splits = splits;
  pg.n_cols = n_cols;
  pg.mode = 2;
  pg.partials = static_cast<float*>(workspace);
  pg.m_half = kDim / 128;

  KvAppendParams pm;
  std::memset(&pm, 0, sizeof pm);
  pm.batch = static_cast<int>(B);
  pm.splits = splits;
  pm.partials = static_cast<const float*>(workspace);
  pm.k_cache = k_cache->data;
  pm.v_cache = v_cache->data;
  pm.fp8 = kv_dtype == MFA_FP8_E4M3;
  pm.k_scale = k_scale;
  pm.v_scale = v_scale;
  pm.positions = static_cast<const int*>(positions->data);
  pm.page_table = paged ? static_cast<const int*>(page_table->data) : nullptr;
  pm.pt_stride = paged ? page_table->stride[0] : 0;
  pm.page_size = page_size;
  pm.max_pages = max_pages;
  pm.num_pages = num_pages;
  pm.cache_bs = k_cache->stride[0];
  pm.cache_ts = k_cache->stride[1];
  pm.cap_tokens = static_cast<int>(cap);

  const cudaError_t e =
      launch_kv_append(twk, twv, tx, pg, pm, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MFA_OK : cuda_fail(e);
}

}  // extern "C"

// ===========================================================================
// Output projection
// ===========================================================================
namespace {

// Stream-K grid: one CTA per SM, at least one per output tile (a CTA's run of
// (tile, k-block) units then crosses at most one tile boundary).
int out_proj_ctas(int64_t k, int64_t n, int sms) {
  const int64_t tiles = n / 128, units = tiles * (k / 64);
  int64_t g = sms < units ? sms : units;
  if (g < tiles) g = tiles;
  return static_cast<int>(g);
}

// Two fp32 partial slots [batch][128] per CTA.
size_t out_proj_ws_bytes(int64_t batch, int64_t k, int64_t n, int sms) {
  return align256(static_cast<size_t>(2) * out_proj_ctas(k, n, sms) * batch * 128 * sizeof(float));
}

}  // namespace

extern "C" {

size_t mfa_output_proj_workspace_size(int batch, int k, int n) {
  if (batch <= 0 || k <= 0 || n <= 0 || k % 64 || n % 128) return 0;
  DeviceInfo d;
  const int rc = current_device(&d);
  if (rc != MFA_OK && rc != MFA_ERR_UNSUPPORTED) return 0;
  return out_proj_ws_bytes(batch, k, n, d.sms);
}

int mfa_output_proj(const mfa_tensor* o, const mfa_tensor* w_o, mfa_tensor* y, void* workspace,
                    size_t workspace_bytes, mfa_stream_t stream) {
  if (!well_formed(o, 2) || !well_formed(w_o, 2) || !well_formed(y, 2)) return MFA_ERR_INVALID_ARG;
  for (const mfa_tensor* t : std::initializer_list<const mfa_tensor*>{o, w_o, y})
    if (t->dtype != MFA_BF16 || t->stride[1] != 1 || t->stride[0] % 8 || !aligned16(t->data))
      return MFA_ERR_INVALID_ARG;
  const int64_t B = o->shape[0], K = o->shape[1], N = w_o->shape[1];
  if (w_o->shape[0] != K || y->shape[0] != B || y->shape[1] != N) return MFA_ERR_INVALID_ARG;
  if (B < 1 || B > 256 || K <= 0 || K % 64 || K > (1 << 20) || N <= 0 || N % 128 ||
      N > (1 << 20))
    return MFA_ERR_UNSUPPORTED;
  DeviceInfo dev;
  int rc = current_device(&dev);
  if (rc != MFA_OK) return rc;
  if (!workspace || workspace_bytes < out_proj_ws_bytes(B, K, N, dev.sms) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255))
    return MFA_ERR_WORKSPACE;
  const int n_cols = static_cast<int>((B + 15) / 16 * 16);
  CUtensorMap tw, ta;
  if (encode_2d(&tw, w_o->data, N, K, w_o->stride[0], 64, 64) != CUDA_SUCCESS ||
      encode_2d(&ta, o->data, K, B, o->stride[0], 64, n_cols) != CUDA_SUCCESS)
    return MFA_ERR_INVALID_ARG;
  QprojParams pg;
  std::memset(&pg, 0, sizeof pg);
  pg.batch = static_cast<int>(B);
  pg.k_blocks = static_cast<int>(K / 64);
  pg.m_total = static_cast<int>(N);
  pg.splits = out_proj_ctas(K, N, dev.sms);  // the stream-K grid
  pg.n_cols = n_cols;
  pg.partials = static_cast<float*>(workspace);
  const cudaError_t e = launch_out_proj(tw, ta, pg, static_cast<__nv_bfloat16*>(y->data),
                                        y->stride[0], reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MFA_OK : cuda_fail(e);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// log-sum-exp merge of partial results over disjoint key ranges
// ---------------------------------------------------------------------------
extern "C" int mfa_lse_merge(const mfa_tensor* o_parts, const mfa_tensor* lse_parts,
                             mfa_tensor* out, mfa_tensor* lse_out, mfa_stream_t stream) {
  if (!well_formed(o_parts, 4) || !well_formed(lse_parts, 3) || !well_formed(out, 3))
    return MFA_ERR_INVALID_ARG;
  if (o_parts->dtype != MFA_F32 || lse_parts->dtype != MFA_F32 ||
      (out->dtype != MFA_BF16 && out->dtype != MFA_F32))
    return MFA_ERR_INVALID_ARG;
  const int64_t S = o_parts->shape[0], B = o_parts->shape[1];
  if (S < 1 || S > (1 << 20) || B < 1 || B > (1 << 20)) return MFA_ERR_INVALID_ARG;
  if (o_parts->shape[2] != kHeads || o_parts->shape[3] != kDim) return MFA_ERR_UNSUPPORTED;
  if (lse_parts->shape[0] != S || lse_parts->shape[1] != B || lse_parts->shape[2] != kHeads ||
      out->shape[0] != B || out->shape[1] != kHeads || out->shape[2] != kDim)
    return MFA_ERR_INVALID_ARG;
  // float4 loads of the parts; float4 (f32) or 8-byte (bf16) stores of the output
  if (o_parts->stride[3] != 1 || o_parts->stride[2] % 4 || o_parts->stride[1] % 4 ||
      o_parts->stride[0] % 4 || !aligned16(o_parts->data))
    return MFA_ERR_INVALID_ARG;
  if (lse_parts->stride[2] != 1) return MFA_ERR_INVALID_ARG;
  const uintptr_t out_align = out->dtype == MFA_F32 ? 15u : 7u;
  if (out->stride[2] != 1 || out->stride[1] % 4 || out->stride[0] % 4 ||
      (reinterpret_cast<uintptr_t>(out->data) & out_align))
    return MFA_ERR_INVALID_ARG;
  if (lse_out && (!well_formed(lse_out, 2) || lse_out->dtype != MFA_F32 ||
                  lse_out->shape[0] != B || lse_out->shape[1] != kHeads ||
                  lse_out->stride[1] != 1))
    return MFA_ERR_INVALID_ARG;
  DeviceInfo dev;
  const int rc = current_device(&dev);
  if (rc != MFA_OK) return rc;
  LseMergeParams p;
  std::memset(&p, 0, sizeof p);
  p.o_parts = static_cast<const float*>(o_parts->data);
  p.o_ss = o_parts->stride[0];
  p.o_sb = o_parts->stride[1];
  p.o_sh = o_parts->stride[2];
  p.lse_parts = static_cast<const float*>(lse_parts->data);
  p.l_ss = lse_parts->stride[0];
  p.l_sb = lse_parts->stride[1];
  p.parts = static_cast<int>(S);
  p.batch = static_cast<int>(B);
  p.out = out->data;
  p.out_f32 = out->dtype == MFA_F32;
  p.out_sb = out->stride[0];
  p.out_sh = out->stride[1];
  p.lse_out = lse_out ? static_cast<float*>(lse_out->data) : nullptr;
  p.lse_sb = lse_out ? lse_out->stride[0] : 0;
  const cudaError_t e = launch_lse_merge(p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MFA_OK : cuda_fail(e);
}
