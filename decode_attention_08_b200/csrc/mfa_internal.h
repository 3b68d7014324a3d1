// mfa_internal.h -- parameter blocks shared by the host launchers and the
// kernels of libmfa.so (not part of the public ABI).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

namespace mfa {

constexpr int kHeads = 64;    // query heads per token
constexpr int kDim = 256;     // head dimension of q and of the shared K / V heads
constexpr int kTile = 128;    // cached tokens per tile = MMA M of the score product

// Decode-attention kernel geometry (bf16 cache).
constexpr int kSlots = 5;                  // TMA ring barriers (the ring uses up to this many slots)
constexpr int kSlotBytes = 128 * 128 * 2;  // one tensor, 128 tokens x 128 dims, bf16
constexpr int kQBytes = kHeads * kDim * 2;
constexpr int kPBytes = kTile * kHeads * 2;  // one 16-bit P block, or an E4M3 pair
constexpr int kDecodeThreads = 384;        // 12 warps: 4 service warps + 2 softmax warpgroups
// all of TMEM: score buffers and O^T accumulators (column map in decode_kernel.cu)
constexpr int kTmemCols = 512;

// One partial (split) result: O [64 heads][256 d] f32, normalised over its range.
constexpr size_t kPartialFloats = static_cast<size_t>(kHeads) * kDim;

struct DecodeParams {
  const int* seq_lens;
  int batch;
  int cap_tokens;       // largest valid sequence length
  int paged;
  int page_size;
  int max_pages;
  int num_pages;
  const int* page_table;
  int64_t pt_stride;    // elements between page-table rows
  int num_splits;       // 0: balanced plan over grid; s > 0: s units per sequence
  int grid;             // CTAs of the attention kernel (the plan depends on it)
  float score_log2;     // softmax_scale * k_scale * log2(e)
  float out_scale;      // v_scale
  void* out;
  int out_f32;
  int64_t out_sb, out_sh;  // out strides (elements) of batch and head; d stride 1
  float* lse_out;          // nullable [B][64]
  int64_t lse_sb;
  float* ws_o;             // [slots][64 heads][256 d] normalised partial outputs
  float* ws_lse;           // [slots][64] their log-sum-exp (natural log)
  // Hand-off between the attention and the combine kernel. Nothing here
  // carries over from one call to the next, so the workspace needs no
  // initialisation: every word below is written by the attention kernel
  // before it lets the combine kernel start (programmatic launch).
  //   ws_plan [B]: balanced plan, bits 0-31 the sequence's first tile in the
  //     batch's tile order, bits 32-63 the batch's total tiles.
  //   ws_flag [slots]: 0 until the slot's partial (and lse) is written in
  //     this call, then 1; each slot's owner CTA clears it first.
  unsigned long long* ws_plan;
  unsigned* ws_flag;
  // [grid][2] where each CTA's tiles began in the previous call on this
  // workspace (first sequence, first tile): a hint for warming L2 before the
  // call's inputs may be read; never trusted for results
  int* ws_hint;
  // limit of the combine kernel's waits for partials (ns); then it records
  // MFA_ERR_TIMEOUT and returns
  unsigned long long wait_ns;
  // grouped-query mode (bf16 cache): q [B, 64, 128], key/value token rows
  // [2 groups][128], heads 0-31 in group 0 and 32-63 in group 1, out [B, 64, 128]
  int gqa;
  // 1: the kernel launched just before this one on the stream is the query
  // projection, which writes only q and lets this grid launch only after its
  // own dependency wait. Every other input and the workspace are then ready at
  // launch; only the q loader waits for the projection grid.
  int q_after_proj;
};

struct QprojParams {
  int batch;
  int k_blocks;          // contraction length / 64
  int m_total;           // output features of this GEMM
  int splits;            // split-K factor (first GEMM)
  int n_cols;            // MMA N (16..256)
  int mode;              // 0: latent GEMM (split-K, fp32 partials, hi/lo latent), 1: up-projection
  float* partials;       // [splits][batch][m_total]  (mode 0)
  int* counters;         // [m_total / 128]           (mode 0)
  __nv_bfloat16* latent; // [2 * batch][m_total], rows 2j / 2j+1 = high part / residual
  __nv_bfloat16* q_out;  // (mode 1 output)
  int64_t q_stride;      // elements between q_out rows
  // mode 2 (key/value append): output tiles m < m_half come from the first
  // weight map (W_k), the others from the second (W_v); partials only
  int m_half;
};

// Key/value append: the rows of the new tokens, merged from the split-K
// partials of the projection and stored into the caches.
struct KvAppendParams {
  int batch;
  int splits;
  const float* partials;   // [splits][batch][2 * kDim] (k features, then v features)
  void* k_cache;
  void* v_cache;
  int fp8;                 // caches hold E4M3 codes (else bf16)
  float k_scale, v_scale;  // FP8: stored code = E4M3(value / scale)
  const int* positions;    // [batch] row of each sequence's new token
  const int* page_table;   // [batch][max_pages], or null for contiguous caches
  int64_t pt_stride;
  int page_size, max_pages, num_pages;
  int64_t cache_bs, cache_ts;  // element strides of a sequence (page, if paged) and a token row
  int cap_tokens;              // contiguous caches: rows per sequence
};

// Both projection GEMMs in one persistent kernel (small batches): split-K
// latent GEMM on m1_tiles x splits CTAs, then the up-projection on m2_tiles
// CTAs, whose weights stream into L2 while the latent is still being formed.
struct QprojFusedParams {
  int batch;
  int k1_blocks, k2_blocks;  // contraction lengths / 64 (hidden, rank)
  int m1_tiles, m2_tiles;    // output tiles of 128 (rank, heads x dim)
  int splits;                // split-K factor of the latent GEMM
  int n1, n2;                // MMA N of the two GEMMs (batch, 2 x batch, padded to 16)
  int rank;                  // latent width
  float* partials;           // [splits][batch][rank]
  int* counters;             // [m1_tiles] split arrivals; counters[kQprojDone]: latent tiles done
  __nv_bfloat16* latent;     // [2 * batch][rank], rows 2j / 2j + 1 = high part / residual
  __nv_bfloat16* q_out;
  int64_t q_stride;
};

// Log-sum-exp merge of attention results over disjoint key ranges.
struct LseMergeParams {
  const float* o_parts;  // [S][B][64][256], d stride 1
  int64_t o_ss, o_sb, o_sh;
  const float* lse_parts;  // [S][B][64], h stride 1
  int64_t l_ss, l_sb;
  int parts, batch;
  void* out;  // [B][64][256] bf16 or f32, d stride 1
  int out_f32;
  int64_t out_sb, out_sh;
  float* lse_out;  // nullable [B][64]
  int64_t lse_sb;
};

constexpr int kQprojDone = 1023;  // counter index of the fused kernel's latent-ready count

}  // namespace mfa
