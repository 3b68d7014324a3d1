// decode_kernel.cu -- MFA decode attention on sm_100a (bf16 or FP8 E4M3 KV cache).
//
// Step-3 page, "Key points -> Architecture": the 64 query heads of a token all
// attend over ONE shared key head and ONE shared value head of dimension 256.
// Because every cached row is shared by all 64 heads, both products of the
// attention are dense contractions and run on the 5th-generation tensor core:
//
//   S^T[t, h] = sum_i K[t, i] * q[h, i]       M = 128 tokens, N = 64 heads, K = 256
//   O^T[i, h] += sum_t V[t, i] * P[h, t]      M = 128 dims (x2), N = 64 heads x (hi, lo), K = 128 tokens
//
// Both are issued "swap-AB" (tokens / head dims on the MMA's M side) so every
// accumulator uses the M = 128 TMEM layout where TMEM lane = matrix row. The
// softmax is computed online over 128-token tiles (running max with lazy
// rescaling, running sum), so each K and V row is read from HBM exactly once.
// The probabilities enter the PV product as an exact-sum pair hi + lo (bf16
// pair, or E4M3 pair with an FP8 cache) in one N = 128 product per step.
//
// CTA = 12 warps (bf16 cache; 20 with an FP8 cache, whose softmax runs in four
// warpgroups of 16 heads), one CTA per SM (persistent):
//   warp 0       TMA producer for the K/V ring (32 KB slots: 5 bf16, 4 FP8)
//   warp 1       TMEM allocator + tcgen05.mma issuer (the whole warp runs the
//                issue loop; elect.sync picks the issuing lane); after the plan
//                it also clears the CTA's partial flags and lets the combine
//                kernel launch
//   warp 2       TMA producer for q (one 32 KB load per sequence segment);
//                with an FP8 cache also the segment publisher
//   warp 3       bf16 cache: segment publisher; FP8 cache: q converter (q to
//                its exact E4M3 pair, a segment ahead)
//   warps 4-7    softmax warpgroup 0: heads 0-31  } thread = one token row of S^T,
//   warps 8-11   softmax warpgroup 1: heads 32-63 } then one head-dim row of O^T
//
// Work split (Flash-Decoding, cited on the DeepSeek-V4 page): the (sequence,
// 128-token tile) pairs of the whole batch are cut into `grid` contiguous,
// equal ranges ("balanced"), or every sequence into `num_splits` equal ranges.
// A range that covers a whole sequence writes the final output. Otherwise it
// writes a partial output normalised over its range plus the range's
// log-sum-exp, and mfa_combine_kernel merges the partials of each split
// sequence in plan order (Flash-Decoding's log-sum-exp combine). The plan
// depends only on seq_lens, num_splits and grid, never on whether the cache is
// paged, so paged and contiguous caches give bit-identical results.
//
// Both kernels are launched with programmatic dependent launch: each may start
// (set up barriers, TMEM, descriptors) while the previous kernel on the stream
// drains, and waits with griddepcontrol.wait before touching any input or output.

#include <cstddef>

#include "mfa_internal.h"
#include "sm100.cuh"

namespace mfa {

// Optional pipeline trace (compile with -DMFA_TRACE; off in the library build):
// clock64() stamps of pipeline events for the first 64 tiles of each CTA.
#ifdef MFA_TRACE
constexpr int kTraceKinds = 16, kTraceTiles = 64, kTraceCtas = 160;
__device__ unsigned long long g_mfa_trace[kTraceCtas * kTraceKinds * kTraceTiles];
#define MFA_TR(kind, idx)                                                                   \
  do {                                                                                      \
    if ((idx) < kTraceTiles && blockIdx.x < kTraceCtas)                                     \
      g_mfa_trace[(blockIdx.x * kTraceKinds + (kind)) * kTraceTiles + (idx)] = clock64();   \
  } while (0)
// absolute (%globaltimer) timeline of both kernels over consecutive calls:
// [call][kernel 0 attention / 1 combine][cta][start, after dependency wait, end]
constexpr int kGtCalls = 8, kGtCtas = 1024;
__device__ unsigned long long g_mfa_gt[kGtCalls * 2 * kGtCtas * 3];
__device__ int g_mfa_cnt[2 * kGtCtas];  // per (kernel, CTA) call counter
#define MFA_GT(kernel, cta, what, call)                                                     \
  do {                                                                                      \
    if ((call) >= 0 && (call) < kGtCalls && (cta) < kGtCtas)                                \
      g_mfa_gt[(((call) * 2 + (kernel)) * kGtCtas + (cta)) * 3 + (what)] = global_timer_ns(); \
  } while (0)
#else
#define MFA_GT(kernel, cta, what, call) \
  do {                                  \
  } while (0)
#define MFA_TR(kind, idx) \
  do {                    \
  } while (0)
#endif

namespace {

// Softmax warpgroups. bf16 cache: two, heads 0-31 | 32-63 (HBM-bound; 168
// registers a thread). FP8 cache: four of 16 heads each: its tile rate is bound
// by the softmax chain, which shorter rows and more warps in flight shorten.
template <bool kFp8>
struct Geo {
  static constexpr int kWG = kFp8 ? 4 : 2;
  static constexpr int kWGHeads = kHeads / kWG;
  static constexpr int kThreads = 128 + 128 * kWG;  // 4 service warps + the softmax warps
  static constexpr int kQGroupWarps = 1 + 4 * kWG;  // FP8 first-segment q conversion group
};

// ---------------------------------------------------------------------------
// shared-memory control block
// ---------------------------------------------------------------------------
template <bool kFp8>
struct __align__(16) DecodeCtrl {
  static constexpr int kWG = Geo<kFp8>::kWG;
  static constexpr int kWGHeads = Geo<kFp8>::kWGHeads;
  uint64_t q_full[2], q_empty[2];  // per q buffer (FP8: two, alternating by segment)
  uint64_t slot_full[kSlots], slot_empty[kSlots];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, o_full;
  uint64_t q_conv[2];  // FP8 cache: q buffer converted to its E4M3 pair
  uint64_t red_full[kWG][2], l_pre[kWG], l_full[kWG];
  uint64_t drain;
  long long t0;    // first global tile of this CTA (balanced plan)
  long long ntot;  // total tiles of the batch (balanced plan)
  uint32_t tmem_base;
  int abort_flag;
  unsigned seg_arrivals;  // softmax-warp arrivals at segment ends (never wraps)
  unsigned q_ready;       // FP8 cache: segments whose q is converted (never wraps)
  float qinv[4];          // FP8 cache: score scale 1/s of segment k at [k & 3]
  unsigned qmax[Geo<kFp8>::kQGroupWarps];  // FP8: per-warp max |q| bits, first segment's conversion
  int b_start, off_start, tiles;
  int L_start;  // length of sequence b_start (balanced plan)
  int scan_warp[Geo<kFp8>::kThreads / 32];
  // vector-loaded (float4): keep 16-byte aligned
  // [tile parity][warpgroup][warp][head]: per-warp tile maxima; at a
  // segment's end the same buffer carries the per-warp row sums
  alignas(16) float red[2][kWG][4][kWGHeads];
  // [tile parity][warpgroup][head]: the running maximum in use for the tile's
  // probabilities (the four warps of a warpgroup store the same values)
  alignas(16) float mv[2][kWG][kWGHeads];
};
static_assert(offsetof(DecodeCtrl<false>, red) % 16 == 0 &&
                  offsetof(DecodeCtrl<false>, mv) % 16 == 0 &&
                  offsetof(DecodeCtrl<true>, red) % 16 == 0 &&
                  offsetof(DecodeCtrl<true>, mv) % 16 == 0,
              "vector-loaded control arrays must be 16-byte aligned");

// Shared memory (1024-byte aligned base): q buffer(s) | ring | P | control.
// bf16: one q buffer, five 32 KB ring slots (HBM-bound: every slot of bytes in
// flight counts) and a 32 KB P tile (probabilities as a bf16 pair hi + lo, two
// 16 KB column blocks). FP8: a 16 KB P tile (an E4M3 pair, two 8 KB blocks)
// and either two q buffers, so the next segment's q is loaded and converted a
// whole segment ahead, with four ring slots; or (kOneQ: every CTA has at most
// one segment, as with a fixed split of no more units than CTAs) one q buffer
// and five slots (measured, E4M3 batch 128 with one unit per sequence: 66.4 ->
// 63.4 us; with several segments per CTA the second q buffer is worth more).
template <bool kFp8, bool kOneQ = !kFp8>
struct SmemLayout {
  static constexpr int kQBufs = (kFp8 && !kOneQ) ? 2 : 1;
  static constexpr int kRing = (kFp8 && !kOneQ) ? 4 : kSlots;
  static constexpr int kPSize = kFp8 ? kPBytes : 2 * kPBytes;
  static constexpr int kQ = 0;
  static constexpr int kRingOff = kQ + kQBufs * kQBytes;
  static constexpr int kP = kRingOff + kRing * kSlotBytes;
  static constexpr int kCtrl = kP + kPSize;
  static constexpr int kBytes = kCtrl + static_cast<int>(sizeof(DecodeCtrl<kFp8>));
};
static_assert(SmemLayout<false>::kBytes <= 227 * 1024 && SmemLayout<true>::kBytes <= 227 * 1024 &&
                  SmemLayout<true, true>::kBytes <= 227 * 1024,
              "shared memory budget");
static_assert(SmemLayout<false>::kRing <= kSlots && SmemLayout<true>::kRing <= kSlots &&
                  SmemLayout<true, true>::kRing <= kSlots,
              "ring barriers");

// bf16 P tile: the hi block and the lo block are 16 KB apart (the LBO of the
// N = 128 MN-major operand); which comes first depends on the segment (below).
constexpr uint32_t kPBlock = kPBytes;

// TMEM column map (512 columns; lane = MMA row, i.e. token row of S^T or
// head-dim row of O^T; column = head).
//   scores: tile g's 64 heads at s_cols(g).
//   O^T, per head-dim half r, the PV product is one N = 128 MMA per step whose
//   columns hold the products with P's hi part and with its lo part; the
//   output is their sum.
//   FP8: 128 columns per half from 128 + 256 r, [hi | lo], single-buffered:
//        a segment's output is read out at its end.
//   bf16: 192 columns per half from 128 + 192 r, [hi of even segments | lo |
//        hi of odd segments]. Even segments write [hi | lo] (P's hi block
//        first), odd segments [lo | hi] (lo block first), so the hi columns are
//        double-buffered by segment while the lo columns are shared: at a
//        segment's end its lo part is added into its hi columns (before the
//        next segment's first PV overwrites lo), and its hi columns are read
//        out while the next segment accumulates into the other hi block.
constexpr uint32_t kColS = 0;

template <bool kFp8>
__device__ __forceinline__ uint32_t o_hi(int seg, int r) {
  return kFp8 ? (r ? 384u : 128u) : 128u + 192u * r + ((seg & 1) ? 128u : 0u);
}
template <bool kFp8>
__device__ __forceinline__ uint32_t o_lo(int seg, int r) {
  return kFp8 ? (r ? 448u : 192u) : 192u + 192u * r;
}
// first column written by the segment's PV products for head-dim half r
template <bool kFp8>
__device__ __forceinline__ uint32_t o_pv(int seg, int r) {
  return kFp8 ? o_hi<kFp8>(seg, r) : 128u + 192u * r + ((seg & 1) ? 64u : 0u);
}
static_assert(128 + 192 * 2 == kTmemCols && 384 + 128 == kTmemCols, "TMEM columns");

// Score buffer of tile g: 64 columns (heads). With an FP8 cache the products
// with q's hi and lo parts accumulate into the same columns (two N = 64
// products per step): the tensor core adds the parts, not the softmax warps,
// whose instruction count bounds the FP8 tile rate.
template <bool kFp8>
__device__ __forceinline__ uint32_t s_cols(uint32_t g) {
  return kColS + (g & 1) * (kFp8 ? 256u : 64u);
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P entries stay <= 2^8

__device__ __forceinline__ int tiles_of(int L) { return (L + kTile - 1) / kTile; }

__device__ __forceinline__ int valid_len(const DecodeParams& p, int b) {
  int L = __ldg(p.seq_lens + b);
  if (L < 0 || L > p.cap_tokens) {
    record_error(5 /* MFA_ERR_BAD_INDEX */);
    return 0;
  }
  return L;
}

// All lanes wait; the outcome is made warp-uniform.
__device__ __forceinline__ uint32_t par(uint32_t u) { return u & 1u; }

// ---------------------------------------------------------------------------
// The per-CTA stream of tiles, walked independently (and identically) by each
// role.
// ---------------------------------------------------------------------------
struct TileInfo {
  int b;            // sequence
  int tile;         // tile index within the sequence
  int L;            // sequence length
  bool seg_first;   // first tile of a segment (run of tiles of one sequence)
  bool seg_last;    // last tile of a segment
  bool cta_last;    // last tile this CTA processes
  int slot;         // partial slot of the segment, -1 when it covers the sequence
  int seg;          // ordinal of the segment among this CTA's segments
  long long gtile;  // global tile index (balanced plan)
};

struct TileStream {
  // scalars copied out of the parameter block at init, so walking the stream
  // never reloads them through memory (the hot loops hold memory-clobbering
  // waits, after which a pointer read would go back out to the cache hierarchy)
  const int* seq_lens;
  int cap_tokens, num_splits, grid, batch;
  int cta;
  int b, tile, L, nt, remaining, seg_lo, seg_hi, seg_ord;
  int segno;  // segments completed so far
  long long gtile;
  int unit, unit_hi;

  // L0: the length of sequence b_start, as the plan read it (balanced plan)
  __device__ void init(const DecodeParams& prm, int b_start, int off_start, int tiles,
                       long long t0, int L0) {
    seq_lens = prm.seq_lens;
    cap_tokens = prm.cap_tokens;
    num_splits = prm.num_splits;
    grid = prm.grid;
    batch = prm.batch;
    cta = blockIdx.x;
    seg_ord = 0;
    segno = 0;
    gtile = t0;
    if (prm.num_splits == 0) {
      remaining = tiles;
      if (remaining > 0) {
        b = b_start;
        L = L0;
        nt = tiles_of(L);
        tile = off_start;
        seg_lo = tile;
        seg_hi = min(nt, seg_lo + remaining);
      }
    } else {
      unit = cta - prm.grid;
      remaining = 0;
      advance_unit();
    }
  }

  // fixed plan: move to the next non-empty unit owned by this CTA
  // (a global load: a shared copy of the lengths costs the FP8 kernel registers
  // it does not have, and reaches only a few loads per CTA)
  __device__ int length(int seq) const {
    int n = __ldg(seq_lens + seq);
    if (n < 0 || n > cap_tokens) {
      record_error(5 /* MFA_ERR_BAD_INDEX */);
      n = 0;
    }
    return n;
  }

  __device__ void advance_unit() {
    const int s = num_splits;
    const int nunits = batch * s;
    for (unit += grid; unit < nunits; unit += grid) {
      b = unit / s;
      const int j = unit % s;
      L = length(b);
      nt = tiles_of(L);
      const int lo = static_cast<int>((static_cast<long long>(j) * nt) / s);
      const int hi = static_cast<int>((static_cast<long long>(j + 1) * nt) / s);
      if (hi > lo) {
        tile = lo;
        seg_lo = lo;
        seg_hi = hi;
        unit_hi = hi;
        remaining = 1;
        return;
      }
    }
    remaining = 0;
  }

  __device__ bool next(TileInfo& t) {
    if (remaining <= 0) return false;
    t.b = b;
    t.tile = tile;
    t.L = L;
    t.seg_first = (tile == seg_lo);
    t.seg_last = (tile == seg_hi - 1);
    t.seg = segno;
    if (t.seg_last) ++segno;
    t.gtile = gtile;
    const bool complete = (seg_lo == 0 && seg_hi == nt);
    if (num_splits == 0) {
      t.slot = complete ? -1 : (2 * cta + (seg_ord == 0 ? 0 : 1));
      ++tile;
      ++gtile;
      --remaining;
      t.cta_last = (remaining == 0);
      if (remaining > 0 && tile == nt) {
        do {
          if (++b >= batch) {  // lengths that disagree with the plan: stop, reported
            record_error(5 /* MFA_ERR_BAD_INDEX */);
            remaining = 0;
            return true;
          }
          L = length(b);
          nt = tiles_of(L);
        } while (nt == 0);
        tile = 0;
        seg_lo = 0;
        seg_hi = min(nt, remaining);
        ++seg_ord;
      }
    } else {
      t.slot = complete ? -1 : unit;
      ++tile;
      if (tile == unit_hi) advance_unit();
      t.cta_last = (remaining == 0);
    }
    return true;
  }
};

// ---------------------------------------------------------------------------
// The partial slots of a split sequence, in plan order.
// ---------------------------------------------------------------------------
struct SplitList {
  int mode;  // 0 balanced, s > 0 fixed
  long long N, G, S;
  int c_first, first_slot;
  bool dense;  // balanced plan with at least one tile per CTA
  int b, nt;
  int count;  // candidates in plan order; slot(i) may be -1 (empty range, fixed plan)

  // balanced plan: the sequence's tiles are [S, S + ntiles) in the global order;
  // CTA c owns tiles [cN/G, (c+1)N/G), so tile t belongs to CTA ((t+1)G - 1) / N.
  __device__ void init_balanced(long long S_, int ntiles, long long Ntot, long long grid) {
    mode = 0;
    N = Ntot;
    G = grid;
    S = S_;
    nt = ntiles;
    dense = N >= G;
    c_first = static_cast<int>(((S + 1) * G - 1) / N);
    const int c_last = static_cast<int>(((S + ntiles) * G - 1) / N);
    const long long start_first = (static_cast<long long>(c_first) * N) / G;
    first_slot = (start_first < S) ? 2 * c_first + 1 : 2 * c_first;
    // with N >= G every CTA owns >= 1 tile; otherwise every CTA owns <= 1 tile
    count = dense ? c_last - c_first + 1 : ntiles;
  }
  __device__ void init_fixed(int seq, int ntiles, int s) {
    mode = s;
    b = seq;
    nt = ntiles;
    count = s;
  }
  __device__ int slot(int i) const {
    if (mode == 0) {
      if (i == 0) return first_slot;
      const long long cc = dense ? c_first + i : ((S + i + 1) * G - 1) / N;
      return static_cast<int>(2 * cc);
    }
    const int lo = static_cast<int>((static_cast<long long>(i) * nt) / mode);
    const int hi = static_cast<int>((static_cast<long long>(i + 1) * nt) / mode);
    return hi > lo ? b * mode + i : -1;
  }
  __device__ int nonempty() const {
    if (mode == 0) return count;
    int n = 0;
    for (int i = 0; i < count; ++i) n += slot(i) >= 0;
    return n;
  }
};

// Partial slots (segments) of the tile's sequence under the plan in use.
__device__ __forceinline__ int segments_of(const DecodeParams& p, const TileInfo& t,
                                           long long ntot) {
  SplitList sl;
  if (p.num_splits == 0) {
    sl.init_balanced(t.gtile - t.tile, tiles_of(t.L), ntot, p.grid);
    return sl.count;
  }
  sl.init_fixed(t.b, tiles_of(t.L), p.num_splits);
  return sl.nonempty();
}

__device__ __forceinline__ void smem_add_release(unsigned* ctr, unsigned v) {
  asm volatile("red.release.cta.shared::cta.add.u32 [%0], %1;" ::"r"(smem_u32(ctr)), "r"(v)
               : "memory");
}

__device__ __forceinline__ unsigned smem_ld_acquire(const unsigned* ctr) {
  unsigned v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(ctr)) : "memory");
  return v;
}

// Waits (bounded, like mbar_wait) until the shared counter reaches `target`.
__device__ __forceinline__ bool wait_count(const unsigned* ctr, unsigned target,
                                           volatile int* abort_flag) {
  if (smem_ld_acquire(ctr) >= target) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 1;; ++it) {
    if (smem_ld_acquire(ctr) >= target) return true;
    if ((it & 255u) == 0) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        record_error(6 /* MFA_ERR_TIMEOUT */);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Publishes a split segment's partial to the combine kernel (one thread, once
// the softmax warps' stores of it are ordered before this thread: their
// release arrivals on the shared counter, acquired by the caller). The release
// store makes those stores visible device-wide with the slot's flag. A segment
// that covers its whole sequence wrote the output itself: nothing to publish.
__device__ __forceinline__ void publish_segment(const DecodeParams& p, const TileInfo& t) {
  if (t.slot < 0) return;
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p.ws_flag + t.slot), "r"(1u)
               : "memory");
}

// ---------------------------------------------------------------------------
// Block-wide plan: total tiles, this CTA's tile range and its first sequence.
// ---------------------------------------------------------------------------
template <int kThreads>
__device__ int block_inclusive_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  int add = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) {
    if (w < warp) add += warp_sums[w];
    tot += warp_sums[w];
  }
  __syncthreads();
  *total = tot;
  return v + add;
}

// Every CTA computes the whole plan (an exclusive scan of the sequences' tile
// counts); CTA c also stores the plan words of sequences b = c (mod grid) for
// the combine kernel.
template <bool kFp8>
__device__ void balanced_plan(const DecodeParams& p, DecodeCtrl<kFp8>& c) {
  constexpr int kThreads = Geo<kFp8>::kThreads;
  const int tid = threadIdx.x;
  const long long G = p.grid;
  long long total = 0;
  long long t0 = 0;
  if (p.batch <= kThreads) {
    // single pass: the whole batch is one chunk
    const int len = tid < p.batch ? valid_len(p, tid) : 0;
    const int n = tiles_of(len);
    int chunk;
    const int incl = block_inclusive_scan<kThreads>(n, c.scan_warp, &chunk);
    total = chunk;
    t0 = (static_cast<long long>(blockIdx.x) * total) / G;
    const long long excl = incl - n;
    if (tid < p.batch && n > 0 && excl <= t0 && t0 < excl + n) {
      c.b_start = tid;
      c.off_start = static_cast<int>(t0 - excl);
      c.L_start = len;
    }
    if (tid < p.batch && tid % p.grid == static_cast<int>(blockIdx.x)) {
      p.ws_plan[tid] = static_cast<unsigned long long>(excl) |
                       (static_cast<unsigned long long>(total) << 32);
      __threadfence();  // before the combine may start (the trigger follows this plan)
    }
  } else {
    for (int base = 0; base < p.batch; base += kThreads) {
      const int b = base + tid;
      const int n = (b < p.batch) ? tiles_of(valid_len(p, b)) : 0;
      int chunk;
      block_inclusive_scan<kThreads>(n, c.scan_warp, &chunk);
      total += chunk;
    }
    t0 = (static_cast<long long>(blockIdx.x) * total) / G;
    long long run = 0;
    for (int base = 0; base < p.batch; base += kThreads) {
      const int b = base + tid;
      const int len = (b < p.batch) ? valid_len(p, b) : 0;
      const int n = tiles_of(len);
      int chunk;
      const int incl = block_inclusive_scan<kThreads>(n, c.scan_warp, &chunk);
      const long long excl = run + incl - n;
      if (b < p.batch && n > 0 && excl <= t0 && t0 < excl + n) {
        c.b_start = b;
        c.off_start = static_cast<int>(t0 - excl);
        c.L_start = len;
      }
      if (b < p.batch && b % p.grid == static_cast<int>(blockIdx.x)) {
        p.ws_plan[b] = static_cast<unsigned long long>(excl) |
                       (static_cast<unsigned long long>(total) << 32);
        __threadfence();  // before the combine may start (the trigger follows this plan)
      }
      run += chunk;
    }
  }
  const long long t1 = (static_cast<long long>(blockIdx.x + 1) * total) / G;
  if (tid == 0) {
    c.tiles = static_cast<int>(t1 - t0);
    c.t0 = t0;
    c.ntot = total;
  }
  __syncthreads();
}

// Fixed split: the next call's L2 warm-up hint, where this CTA's first unit
// begins (out of line: it runs once, by one thread).
__device__ __noinline__ void fixed_plan_hint(const int* seq_lens, int cap_tokens, int num_splits,
                                             int* hint, bool has_units) {
  int hb = -1, ht = 0;
  if (has_units) {
    const int b = static_cast<int>(blockIdx.x) / num_splits;
    const int j = static_cast<int>(blockIdx.x) % num_splits;
    const int L = __ldg(seq_lens + b);
    const int nt = (L < 0 || L > cap_tokens) ? 0 : tiles_of(L);  // (reported by the plan)
    const int lo = static_cast<int>((static_cast<long long>(j) * nt) / num_splits);
    const int hi = static_cast<int>((static_cast<long long>(j + 1) * nt) / num_splits);
    if (hi > lo) {
      hb = b;
      ht = lo;
    }
  }
  hint[2 * blockIdx.x] = hb;
  hint[2 * blockIdx.x + 1] = ht;
}

// ---------------------------------------------------------------------------
// warp-level "reduce-scatter": on entry each lane has 32 per-head values of its
// own row; on exit lane l holds the reduction over all 32 lanes for head l.
// ---------------------------------------------------------------------------
template <bool kMax, int N, int MASK, int NV>
__device__ __forceinline__ void rs_step(float (&v)[NV], int lane) {
  const bool upper = (lane & MASK) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = upper ? v[i] : v[i + N / 2];
    const float keep = upper ? v[i + N / 2] : v[i];
    const float recv = __shfl_xor_sync(0xffffffffu, send, MASK);
    v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
}

// NV = 32: lane l returns the reduction of value l over the 32 lanes. NV = 16:
// lanes 2j and 2j + 1 both return the reduction of value j.
template <bool kMax, int NV>
__device__ __forceinline__ float reduce_scatter(float (&v)[NV], int lane) {
  if constexpr (NV == 32) {
    rs_step<kMax, 32, 16>(v, lane);
    rs_step<kMax, 16, 8>(v, lane);
    rs_step<kMax, 8, 4>(v, lane);
    rs_step<kMax, 4, 2>(v, lane);
    rs_step<kMax, 2, 1>(v, lane);
    return v[0];
  } else {
    static_assert(NV == 16, "16 or 32 values per lane");
    rs_step<kMax, 16, 16>(v, lane);
    rs_step<kMax, 8, 8>(v, lane);
    rs_step<kMax, 4, 4>(v, lane);
    rs_step<kMax, 2, 2>(v, lane);
    const float o = __shfl_xor_sync(0xffffffffu, v[0], 1);
    return kMax ? fmaxf(v[0], o) : v[0] + o;
  }
}

// Ring items per tensor and tile: bf16 K or V tiles take two 32 KB slots (head
// dims 0-127, 128-255); an E4M3 tile fits one slot (its two 16 KB halves).
template <bool kFp8>
constexpr uint32_t kItemsPerTensor = kFp8 ? 1u : 2u;

// Index, in producer order, of the first ring item holding V of the CTA's j-th
// tile: items go K0 | K1 V0 | K2 V1 | ... | K(T-1) V(T-2) | V(T-1).
template <bool kFp8>
__device__ __forceinline__ uint32_t v_item(uint32_t j, bool cta_last) {
  constexpr uint32_t n = kItemsPerTensor<kFp8>;
  return cta_last ? 2u * n * j + n : 2u * n * j + 2u * n;
}

// Page ids of 32 consecutive logical pages of one sequence, one per lane of the
// producer warp, so a TMA issue never waits on a dependent page-table load:
// a refill reads up to 32 entries in parallel (never past the sequence's last
// page, as the interface promises) and ids are taken by warp shuffle.
struct PageWindow {
  int b = -1, base = 0, val = 0;
  // id of logical page `lp` (per lane) of sequence `seq`; [lo, hi] (warp-uniform,
  // hi - lo < 32) bounds the pages the warp asks for in this call
  __device__ __forceinline__ int get(const int* table, int64_t stride, int seq, int lo, int hi,
                                     int lp, int npages, int lane) {
    if (seq != b || lo < base || hi >= base + 32) {  // warp-uniform
      b = seq;
      base = lo;
      const int mine = base + lane;
      val = mine < npages ? __ldg(table + static_cast<int64_t>(seq) * stride + mine) : 0;
    }
    return __shfl_sync(0xffffffffu, val, lp - base);
  }
};

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

// FP8 cache, per segment: q (bf16, 64 heads x 256 dims, as TMA wrote it: four
// 8 KB regions of 64 dims, 128-byte rows with the 128-byte swizzle) becomes two
// E4M3 operands whose sum is q * s exactly (s a power of two putting max|q*s|
// in [128, 256); bf16's 8 significant bits split into two 4-bit parts):
// dims half c (0, 1) -> hi at 16 KB * c, lo at 16 KB * c + 8 KB, each 64 rows
// of 128 dims (128-byte rows, 128-byte swizzle). Returns 1 / s.

// max |q| over the tile (all lanes get it)
__device__ __forceinline__ float q_max_abs(uint32_t base, int lane) {
  uint32_t m = 0;
#pragma unroll 8
  for (int i = lane; i < kQBytes / 16; i += 32) {
    const uint4 v = ld_shared_v4(base + i * 16);
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu),
                             __vmaxu2(v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu)));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = __vmaxu2(m, __shfl_xor_sync(0xffffffffu, m, o));
  const uint32_t top = (m >> 16) > (m & 0xFFFFu) ? (m >> 16) : (m & 0xFFFFu);
  return __uint_as_float(top << 16);
}

// Score scale of a q whose largest |element| has the bf16 bits `top`:
// s = 2^(7 - E) with max|q| in [2^E, 2^(E+1)); the exponent field is clamped
// so that s and 1/s stay normal floats (an all-zero q takes any scale).
__device__ __forceinline__ void q_scale(uint32_t top, float& s, float& inv_s) {
  int ebits = static_cast<int>(((top << 16) >> 23) & 0xFF);
  ebits = ebits < 8 ? 8 : (ebits > 253 ? 253 : ebits);
  s = __uint_as_float(static_cast<uint32_t>(261 - ebits) << 23);
  inv_s = __uint_as_float(static_cast<uint32_t>(ebits - 7) << 23);
}

// The conversion works on units of 16 dims of one head and dims half: 32 bytes
// of bf16 q in, 16 bytes of hi and 16 bytes of lo E4M3 out. The loaded q of a
// head and dims half is two 128-byte rows (dims 0-63 | 64-127 of the half,
// 8 KB apart, 16-byte chunks swizzled by the head); its E4M3 pair takes the
// same two rows, hi then lo. Unit m (0-7) reads chunks 2m, 2m+1 of that span
// and writes chunk m of each row, so a head's units are converted only after
// all eight have read their input. A thread takes four consecutive units (one
// row half) and holds their input in registers; the code is one short rolled
// loop: it runs once per segment, where a long unrolled body would mostly wait
// for instruction fetch.
constexpr int kQUnits = 2 * kHeads * 8;  // head x dims half x 16-dim unit
constexpr int kQUnitsPerThread = 4;

// Loads the input of units [4 t, 4 t + 4): head h = t / 4, dims half c = (t / 2) & 1,
// units 4 (t & 1) .. + 3 (input row k = t & 1).
__device__ __forceinline__ void q_load_units(uint32_t base, int t, uint4 (&in)[8]) {
  const int h = t >> 2, c = (t >> 1) & 1, k = t & 1, sw = h & 7;
  const uint32_t row = base + (2 * c + k) * 8192 + h * 128;
#pragma unroll
  for (int j = 0; j < 8; ++j) in[j] = ld_shared_v4(row + ((j ^ sw) << 4));
}

__device__ __forceinline__ uint32_t q_units_max(const uint4 (&in)[8]) {
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    m = __vmaxu2(m, __vmaxu2(__vmaxu2(in[j].x & 0x7FFF7FFFu, in[j].y & 0x7FFF7FFFu),
                             __vmaxu2(in[j].z & 0x7FFF7FFFu, in[j].w & 0x7FFF7FFFu)));
  return m;
}

// Writes the E4M3 pairs of the units loaded by q_load_units(base, t, in).
__device__ __forceinline__ void q_store_units(uint32_t base, int t, float s, uint4 (&in)[8]) {
  const int h = t >> 2, c = (t >> 1) & 1, sw = h & 7;
  const uint32_t hi_row = base + c * 16384 + h * 128;
  const uint32_t lo_row = hi_row + 8192;
#pragma unroll 1
  for (int q = 0; q < kQUnitsPerThread; ++q) {
    const int m = 4 * (t & 1) + q;  // output chunk: dims 16m..16m+15 of the half
    uint32_t w[8];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint4 v = in[u];
      const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; e += 2) {
        // four bf16 -> two hi/lo pairs
        const uint32_t p0 = split_e4m3x2(__uint_as_float(wd[e] << 16) * s,
                                         __uint_as_float(wd[e] & 0xFFFF0000u) * s);
        const uint32_t p1 = split_e4m3x2(__uint_as_float(wd[e + 1] << 16) * s,
                                         __uint_as_float(wd[e + 1] & 0xFFFF0000u) * s);
        w[4 * u + e / 2] = (p0 & 0xFFFFu) | (p1 << 16);          // hi bytes
        w[4 * u + 2 + e / 2] = (p0 >> 16) | (p1 & 0xFFFF0000u);  // lo bytes
      }
    }
    st_shared_v4(hi_row + ((m ^ sw) << 4), w[0], w[1], w[4], w[5]);
    st_shared_v4(lo_row + ((m ^ sw) << 4), w[2], w[3], w[6], w[7]);
#pragma unroll
    for (int j = 0; j < 6; ++j) in[j] = in[j + 2];  // next unit's input to in[0..1]
  }
}

// q of a segment to its exact E4M3 pair, in place, by one warp; returns 1/s.
__device__ __forceinline__ float q_to_e4m3(uint32_t base, int lane) {
  float s, inv_s;
  q_scale(__float_as_uint(q_max_abs(base, lane)) >> 16, s, inv_s);
  // rounds of 32 threads x 4 units = 16 whole (head, dims half) spans
#pragma unroll 1
  for (int r = 0; r < kQUnits / (32 * kQUnitsPerThread); ++r) {
    uint4 in[8];
    const int t = r * 32 + lane;
    q_load_units(base, t, in);
    __syncwarp();  // both halves of each span read before either writes
    q_store_units(base, t, s, in);
  }
  return inv_s;
}

// The same conversion by warp 3 and the softmax warps together, for a CTA's
// first segment (its first product waits for it, and the softmax warps would
// otherwise wait for that product). gtid = thread index - 96; threads below
// kQUnits / 4 take four units each. Every thread of the group calls it exactly
// once, also after a failed wait (work = false): it holds two barriers
// (named barrier 1) of the whole group, the first of which also orders every
// read of q before the in-place writes. The softmax warps only arrive at the
// second; warp 3 waits there, then publishes.
constexpr int kQGroupWarps = Geo<true>::kQGroupWarps;
constexpr int kQGroupThreads = 32 * kQGroupWarps;
static_assert(kQGroupThreads * kQUnitsPerThread >= kQUnits, "group covers q in one round");
__device__ __forceinline__ float q_to_e4m3_group(uint32_t base, int gtid, bool work, bool publisher,
                                                 unsigned* part) {
  const bool mine = work && gtid < kQUnits / kQUnitsPerThread;
  uint4 in[8];
  uint32_t m = 0;
  if (mine) {
    q_load_units(base, gtid, in);
    m = q_units_max(in);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = __vmaxu2(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((gtid & 31) == 0) part[gtid >> 5] = (m >> 16) > (m & 0xFFFFu) ? (m >> 16) : (m & 0xFFFFu);
  asm volatile("bar.sync 1, %0;" ::"n"(kQGroupThreads) : "memory");
  uint32_t top = 0;
#pragma unroll
  for (int w = 0; w < kQGroupWarps; ++w) top = part[w] > top ? part[w] : top;
  float s, inv_s;
  q_scale(top, s, inv_s);
  if (mine) q_store_units(base, gtid, s, in);
  fence_proxy_async_smem();
  if (publisher)
    asm volatile("bar.sync 1, %0;" ::"n"(kQGroupThreads) : "memory");
  else
    asm volatile("bar.arrive 1, %0;" ::"n"(kQGroupThreads) : "memory");
  return inv_s;
}

constexpr int kCombineHeads = 16;  // heads per CTA
constexpr int kCombineDims = 16;   // head-dim elements per thread (kDim / 16 threads per head)

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* w) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(w) : "memory");
  return v;
}

// Waits (bounded by limit_ns) until the flag is set; false after the limit
// (MFA_ERR_TIMEOUT recorded). Polls with acquire loads, ordering the caller's
// reads of the partial after the flag.
__device__ bool wait_flag(const unsigned* f, unsigned long long limit_ns) {
  if (ld_acquire_u32(f) != 0) return true;
  const uint64_t t0 = global_timer_ns();
  while (ld_acquire_u32(f) == 0) {
    if (global_timer_ns() - t0 > limit_ns) {
      record_error(6 /* MFA_ERR_TIMEOUT */);
      return false;
    }
  }
  return true;
}

// 16 consecutive output elements of (b, h) from d0 (16-byte vector stores
// when the address allows).
__device__ __forceinline__ void store_out16(const DecodeParams& p, int b, int h, int d0,
                                            const float* v) {
  const int64_t off = static_cast<int64_t>(b) * p.out_sb + static_cast<int64_t>(h) * p.out_sh + d0;
  if (p.out_f32) {
    float* dst = static_cast<float*>(p.out) + off;
    if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
      for (int j = 0; j < kCombineDims / 4; ++j)
        reinterpret_cast<float4*>(dst)[j] = make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    } else {
#pragma unroll
      for (int j = 0; j < kCombineDims; ++j) dst[j] = v[j];
    }
  } else {
    __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + off;
    if ((reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
#pragma unroll
      for (int j = 0; j < kCombineDims / 8; ++j)
        reinterpret_cast<uint4*>(dst)[j] =
            make_uint4(pack_bf16x2(v[8 * j], v[8 * j + 1]), pack_bf16x2(v[8 * j + 2], v[8 * j + 3]),
                       pack_bf16x2(v[8 * j + 4], v[8 * j + 5]), pack_bf16x2(v[8 * j + 6], v[8 * j + 7]));
    } else {
#pragma unroll
      for (int j = 0; j < kCombineDims; ++j) dst[j] = __float2bfloat16_rn(v[j]);
    }
  }
}

// Merges the partials of split sequence b for head h, head-dim elements
// d0 .. d0 + 15, in plan order (up to four per round trip), and writes the
// output and (d0 == 0) the log-sum-exp. The partials must be visible to the
// caller (acquired after the sequence's last arrival).
// kCombineBatch: partials loaded per round trip
template <int kCombineBatch>
__device__ __forceinline__ void merge_head_part(const DecodeParams& p, int b, const SplitList& sl,
                                                int h, int d0) {
  // online merge: running max m, running weight sum l, running weighted sums v
  float v[kCombineDims];
  float m = -INFINITY, l = 0.f;
#pragma unroll
  for (int j = 0; j < kCombineDims; ++j) v[j] = 0.f;
  for (int i = 0; i < sl.count; i += kCombineBatch) {
    int slot[kCombineBatch];
    bool any = false;
#pragma unroll
    for (int k = 0; k < kCombineBatch; ++k) {
      slot[k] = i + k < sl.count ? sl.slot(i + k) : -1;
      any |= slot[k] >= 0;
    }
    if (!any) continue;  // empty units of a fixed split
    float e[kCombineBatch];
    float4 o[kCombineBatch][kCombineDims / 4];
#pragma unroll
    for (int k = 0; k < kCombineBatch; ++k) {
      const int sk = slot[k] < 0 ? 0 : slot[k];
      const float4* src = reinterpret_cast<const float4*>(
          p.ws_o + static_cast<int64_t>(sk) * kPartialFloats + static_cast<int64_t>(h) * kDim + d0);
      e[k] = slot[k] >= 0 ? __ldcg(p.ws_lse + static_cast<int64_t>(sk) * kHeads + h) : -INFINITY;
#pragma unroll
      for (int j = 0; j < kCombineDims / 4; ++j)
        o[k][j] = slot[k] >= 0 ? __ldcg(src + j) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mn = m;
#pragma unroll
    for (int k = 0; k < kCombineBatch; ++k) mn = fmaxf(mn, e[k]);  // finite: one slot is valid
    const float c = ex2_approx((m - mn) * kLog2e);
    l *= c;
#pragma unroll
    for (int j = 0; j < kCombineDims; ++j) v[j] *= c;
#pragma unroll
    for (int k = 0; k < kCombineBatch; ++k) {
      const float w = ex2_approx((e[k] - mn) * kLog2e);
      l += w;
#pragma unroll
      for (int j = 0; j < kCombineDims / 4; ++j) {
        v[4 * j] += w * o[k][j].x;
        v[4 * j + 1] += w * o[k][j].y;
        v[4 * j + 2] += w * o[k][j].z;
        v[4 * j + 3] += w * o[k][j].w;
      }
    }
    m = mn;
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int j = 0; j < kCombineDims; ++j) v[j] *= inv;
  store_out16(p, b, h, d0, v);
  if (p.lse_out && d0 == 0) p.lse_out[b * p.lse_sb + h] = m + lg2_approx(l) * kLn2;
}

// The split list of sequence b (nt > 0 tiles): from its plan word (balanced
// plan), or from the fixed split.
__device__ __forceinline__ SplitList split_list_of(const DecodeParams& p, int b, int nt) {
  SplitList sl;
  if (p.num_splits == 0) {
    const unsigned long long word = __ldcg(p.ws_plan + b);
    sl.init_balanced(static_cast<long long>(word & 0xffffffffull), nt,
                     static_cast<long long>(word >> 32), p.grid);
  } else {
    sl.init_fixed(b, nt, p.num_splits);
  }
  return sl;
}

}  // namespace

// A finished segment's output, read by one softmax warp: its 32 heads
// (columns from tcol) for head-dim rows `row` and 128 + `row` (O^T rows in
// TMEM lanes), scaled per head by the output scale that lane `head` holds in
// ev; the output (slot < 0) or the partial of a
// split sequence (layout [slot][head][d]: a warp writes 128 contiguous bytes
// per head). The accumulator of half r is the hi columns hi_r plus, when
// add_lo, the lo columns lo_r (a bf16 segment whose lo part was already added
// into its hi columns passes add_lo = false). Out of line: it runs once per
// segment, and its code inlined in the softmax loop (two or three copies)
// measurably slowed that loop.
template <int W>
__device__ __forceinline__ void tmem_ldw(uint32_t taddr, uint32_t (&r)[W]) {
  if constexpr (W == 32)
    tmem_ld32(taddr, r);
  else
    tmem_ld16(taddr, r);
}

template <bool kFp8>
__device__ __noinline__ void segment_out(float* ws_o, void* out, int out_f32, int64_t out_sb,
                                         int64_t out_sh, int slot, int b, uint32_t tcol,
                                         uint32_t hi0, uint32_t hi1, uint32_t lo0, uint32_t lo1,
                                         bool add_lo, int row, int hbase, float ev, int gqa) {
  constexpr int W = Geo<kFp8>::kWGHeads;  // this warp's heads (columns)
#pragma unroll 1
  for (int half = 0; half < 2; ++half) {
    // grouped-query mode: this warpgroup's heads form one group, whose output
    // is O^T's head-dim half of that group (out rows of 128 dims)
    if (gqa && half != (hbase >> 5)) continue;
    const int d = gqa ? row : half * 128 + row;
    uint32_t r[W];
    tmem_ldw<W>(tcol + (half ? hi1 : hi0), r);
    if (add_lo) {  // O = (V P_hi) + (V P_lo)
      uint32_t r2[W];
      tmem_ldw<W>(tcol + (half ? lo1 : lo0), r2);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < W; ++j)
        r[j] = __float_as_uint(__uint_as_float(r[j]) + __uint_as_float(r2[j]));
    } else {
      tmem_wait_ld();
    }
    // per head j: the output scale held by lane j (a shuffle; a shared-memory
    // copy measured slower: it cost the 168-register kernel a spill)
#pragma unroll
    for (int j = 0; j < W; ++j)
      r[j] = __float_as_uint(__uint_as_float(r[j]) * __shfl_sync(0xffffffffu, ev, j));
    if (slot >= 0) {
      float* dst = ws_o + static_cast<int64_t>(slot) * kPartialFloats +
                   static_cast<int64_t>(hbase) * kDim + d;
#pragma unroll
      for (int j = 0; j < W; ++j) dst[j * kDim] = __uint_as_float(r[j]);
    } else if (out_f32) {
      float* dst = static_cast<float*>(out) + b * out_sb + hbase * out_sh + d;
#pragma unroll
      for (int j = 0; j < W; ++j) dst[j * out_sh] = __uint_as_float(r[j]);
    } else {
      __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(out) + b * out_sb + hbase * out_sh + d;
#pragma unroll
      for (int j = 0; j < W; ++j) dst[j * out_sh] = __float2bfloat16_rn(__uint_as_float(r[j]));
    }
  }
}

// ===========================================================================
// the attention kernel
// ===========================================================================
template <bool kPaged, bool kFp8, bool kOneQ>
__global__ void __launch_bounds__(Geo<kFp8>::kThreads, 1)
    mfa_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  // 1024-byte alignment (the 128-byte swizzle atoms); checked below
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  using L = SmemLayout<kFp8, kOneQ>;
  constexpr uint32_t kS = L::kRing;  // ring slots
  // q buffer of the k-th segment (k & 1 with two buffers) and its phase parity
  constexpr bool kTwoQ = L::kQBufs == 2;
  uint8_t* sQ = smem + L::kQ;
  uint8_t* sRing = smem + L::kRingOff;
  uint8_t* sP = smem + L::kP;
  constexpr int kWG = Geo<kFp8>::kWG;
  constexpr int kWGHeads = Geo<kFp8>::kWGHeads;
  constexpr int kThreads = Geo<kFp8>::kThreads;
  DecodeCtrl<kFp8>& c = *reinterpret_cast<DecodeCtrl<kFp8>*>(smem + L::kCtrl);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  if (smem_u32(smem_raw) & 1023u) {  // never expected: report, do nothing
    if (tid == 0) record_error(2 /* MFA_ERR_UNSUPPORTED */);
    return;
  }

  if (tid == 0) MFA_TR(9, 0);
#ifdef MFA_TRACE
  const unsigned long long gt_start = global_timer_ns();
#endif

  // ---- setup (independent of the previous kernel's results) ----------------
  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.q_full[i], 1);
      mbar_init(&c.q_empty[i], 1);
      mbar_init(&c.q_conv[i], 1);
    }
    for (int i = 0; i < static_cast<int>(kS); ++i) {
      mbar_init(&c.slot_full[i], 1);
      mbar_init(&c.slot_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.s_empty[i], 4 * kWG);
    }
    for (int w = 0; w < kWG; ++w) {
      mbar_init(&c.red_full[w][0], 4);
      mbar_init(&c.red_full[w][1], 4);
      mbar_init(&c.l_pre[w], 4);
      mbar_init(&c.l_full[w], 4);
    }
    mbar_init(&c.p_full, 4 * kWG);
    mbar_init(&c.o_full, 1);
    mbar_init(&c.drain, 1);
    c.abort_flag = 0;
    c.seg_arrivals = 0;
    c.q_ready = 0;
    c.b_start = 0;
    c.off_start = 0;
    c.L_start = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (!kFp8 && p.gqa) {
    // Grouped-query mode: group g's 32 heads hold their q (128 dims) in head
    // dims 128 g .. 128 g + 127 of the 256-wide operand rows and zeros in the
    // other half, so the score product over 256 dims is the group's own 128-dim
    // product (q region r = dims 64 r .. 64 r + 63, 128-byte rows). The zero
    // rows are written once here; q loads never touch them.
    for (int i = tid; i < 1024; i += kThreads) {
      const int r = i >> 8, j = i & 255;
      const int row = (r < 2 ? 32 : 0) + (j >> 3);
      st_shared_v4(smem_u32(sQ) + r * 8192 + row * 128 + (j & 7) * 16, 0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }

  // ---- warm L2 while the previous kernel finishes ---------------------------
  // This call's inputs may not be read before the dependency wait, but an L2
  // prefetch changes no result: the first K/V tiles this CTA took in the
  // previous call on this workspace (a decode loop's plan barely moves from
  // step to step) are fetched while HBM idles under the previous kernel's tail.
  if (!kPaged && warp == 0 && lane == 0) {
    const int hb = *reinterpret_cast<volatile const int*>(p.ws_hint + 2 * blockIdx.x);
    const int ht = *reinterpret_cast<volatile const int*>(p.ws_hint + 2 * blockIdx.x + 1);
    if (hb >= 0 && hb < p.batch && ht >= 0 && ht < (p.cap_tokens + kTile - 1) / kTile) {
      for (int i = 0; i < 2; ++i)
        for (int ch = 0; ch < (kFp8 ? 1 : 2); ++ch) {
          tma_prefetch_4d(&tm_k, 0, (ht + i) * kTile, 2 * ch, hb);
          tma_prefetch_4d(&tm_v, 0, (ht + i) * kTile, 2 * ch, hb);
        }
    }
  }

  // ---- plan (reads seq_lens: after the previous kernel has completed, or at
  // once after the query projection, which launched this grid only after
  // every kernel before it had completed) ----------------------------------
  if (!p.q_after_proj) griddep_wait();
  if (tid == 0) MFA_TR(10, 0);
#ifdef MFA_TRACE
  const int gt_call = blockIdx.x < kGtCtas ? *reinterpret_cast<volatile int*>(&g_mfa_cnt[blockIdx.x]) : -1;
  if (tid == 0) {
    MFA_GT(0, blockIdx.x, 1, gt_call);
    if (gt_call >= 0 && gt_call < kGtCalls && blockIdx.x < kGtCtas)
      g_mfa_gt[((gt_call * 2) * kGtCtas + blockIdx.x) * 3] = gt_start;
  }
#endif
  if (p.num_splits == 0) {
    balanced_plan(p, c);  // its plan words are fenced by their writers
  } else if (tid == 0) {
    c.tiles = static_cast<int>(blockIdx.x) < p.batch * p.num_splits ? -1 : 0;
    c.t0 = 0;
    c.ntot = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (tid == 0) MFA_TR(10, 1);

  // Set-up off the loaders' path, by the MMA warp (whose first products wait
  // for q and the first K tile anyway): this CTA's partial slots (balanced
  // plan: 2c and 2c + 1; fixed split: units c, c + grid, ...) start the call
  // with cleared flags, the next call's L2 warm-up hint is written, and then
  // the combine kernel may start: it starts once every CTA of this grid has
  // passed the trigger (one thread's suffices for its CTA), so it never sees
  // a flag of an earlier call or a plan word not yet written (those were
  // fenced by their writers before the barrier above).
  if (warp == 1) {
    if (p.num_splits == 0) {
      if (lane < 2) p.ws_flag[2 * blockIdx.x + lane] = 0u;
      if (lane == 0) {
        p.ws_hint[2 * blockIdx.x] = c.tiles > 0 ? c.b_start : -1;
        p.ws_hint[2 * blockIdx.x + 1] = c.off_start;
      }
    } else {
      const long long units = static_cast<long long>(p.batch) * p.num_splits;
      for (long long u = blockIdx.x + static_cast<long long>(lane) * p.grid; u < units;
           u += 32LL * p.grid)
        p.ws_flag[u] = 0u;
      if (lane == 0)
        fixed_plan_hint(p.seq_lens, p.cap_tokens, p.num_splits, p.ws_hint, c.tiles != 0);
    }
    __threadfence();
    __syncwarp();
    griddep_launch_dependents();
  }

  volatile int* abort_flag = &c.abort_flag;
  const uint32_t tmem = c.tmem_base;

  if (c.tiles == 0) {
    // no work for this CTA
  } else if (warp == 0) {
    // ======================= K/V producer ===================================
    const uint64_t policy = l2_policy_evict_first();
    TileStream ks;
    ks.init(p, c.b_start, c.off_start, c.tiles, c.t0, c.L_start);
    uint32_t item = 0;
#ifdef MFA_TRACE
    int ntr[2] = {0, 0};
#endif
    PageWindow win;
    // paged-cache fields held in registers for the whole loop; page sizes are
    // powers of two, so every page split is a shift or a mask
    const int ps = kPaged ? p.page_size : kTile;
    const int pshift = __ffs(ps) - 1;
    const int rshift = pshift < 7 ? pshift : 7;  // log2 tokens per box (one page, or one tile)
    const int rows = 1 << rshift;
    const int nsub = kTile >> rshift;
    const int num_pages = p.num_pages;
    const int* page_table = p.page_table;
    const int64_t pt_stride = p.pt_stride;
    // bf16: per item (head dims 0-127 or 128-255) two boxes of 64 dims x rows
    // (or one 4-D box of both); FP8: one item per tensor, two boxes of 128
    // dims x rows, one per 16 KB half of the slot
    constexpr int kBoxes = 2;
    constexpr int kBoxDims = kFp8 ? 128 : 64;
    const bool four_d = rshift == 7;  // contiguous, or pages of >= 128 tokens

    // Sub-pages of a tile (paged caches): lane j < nbox loads sub-page j (a
    // page, or the part of a >= 128-token page under the tile) and holds its
    // page id. K and V share the page table, so a tile is looked up once.
    auto lookup = [&](const TileInfo& t, int& page, int& nbox) {
      page = 0;
      nbox = 1;
      if (kPaged) {
        const int t0 = t.tile * kTile;
        const int live = (t.L - t0 + rows - 1) >> rshift;
        nbox = live < nsub ? live : nsub;
        const int first = t0 >> pshift;
        page = win.get(page_table, pt_stride, t.b, first, first + nbox - 1,
                       first + (lane < nbox ? lane : 0), (t.L + ps - 1) >> pshift, lane);
        if (lane < nbox && (page < 0 || page >= num_pages)) {
          record_error(5 /* MFA_ERR_BAD_INDEX */);
          page = 0;
        }
      }
    };
    // The producer's steady-state code is kept to one short copy (K and V go
    // through the same issue site): it runs seldom next to the consumers' hot
    // loops, so each instruction-cache line it touches tends to be refetched
    // from L2, slowly while HBM is saturated.
    TileInfo tk, tv;       // the next K tile; the tile whose V is pending
    int pgk = 0, nbk = 1;  // lookups of tk
    int pgv = 0, nbv = 1;  // lookups of tv
    bool have_k = ks.next(tk), have_v = false;
    if (have_k) lookup(tk, pgk, nbk);
    // ring order K0 K1 V0 K2 V1 ... K(T-1) V(T-2) V(T-1): round i issues K_i
    // (phase 0), then V_(i-1) (phase 1), then moves to the next tile
    int phase = 0;
    while (have_k || have_v) {
      const bool is_k = phase == 0;
      if (is_k ? have_k : have_v) {
        const TileInfo t = is_k ? tk : tv;
        const int page = is_k ? pgk : pgv;
        const int nbox = is_k ? nbk : nbv;
        const CUtensorMap* map = is_k ? &tm_k : &tm_v;
#ifdef MFA_TRACE
        const int kind = is_k ? 0 : 1;
#endif
        const int t0 = t.tile * kTile;
        const uint32_t bytes =
            four_d ? kSlotBytes : static_cast<uint32_t>(nbox * rows * 128 * kBoxes);
        bool ok = true;
        for (int half = 0; half < static_cast<int>(kItemsPerTensor<kFp8>) && ok; ++half) {
          const uint32_t slot = item % kS;
          ok = mbar_wait_warp(&c.slot_empty[slot], par(item / kS) ^ 1u, abort_flag);
          if (!ok) break;
          uint8_t* dst = sRing + slot * kSlotBytes;
          if (lane == 0) {
            if (half == 0) MFA_TR(kind, ntr[kind]);
            mbar_arrive_expect_tx(&c.slot_full[slot], bytes);
          }
          __syncwarp();
          if (lane < nbox) {
            const int outer = kPaged ? page : t.b;
            if (four_d) {
              // the map views each token row as 4 chunks of 64 dims (chunk
              // stride 128 B) after the token dimension: the box lands as
              // [chunk][128 tokens][128 B]
              tma_load_4d(dst, map, &c.slot_full[slot], 0, kPaged ? (t0 & (ps - 1)) : t0,
                          kFp8 ? 0 : 2 * half, outer, policy);
            } else {
              const int tok = t0 + (lane << rshift);
              for (int r = 0; r < kBoxes; ++r)
                tma_load_3d(dst + r * (kSlotBytes / 2) + lane * rows * 128, map,
                            &c.slot_full[slot], (kBoxes * half + r) * kBoxDims,
                            kPaged ? (tok & (ps - 1)) : tok, outer, policy);
            }
          }
          __syncwarp();
          if (lane == 0) MFA_TR(13, item);
          ++item;
        }
        if (!ok) break;
#ifdef MFA_TRACE
        if (lane == 0) MFA_TR(14 + kind, ntr[kind]);  // both halves issued
        ++ntr[kind];
#endif
      }
      if (!is_k) {
        // end of the round: this K tile's V is next; fetch the following K tile
        have_v = have_k;
        if (have_k) {
          tv = tk;
          pgv = pgk;
          nbv = nbk;
          have_k = ks.next(tk);
          if (have_k) lookup(tk, pgk, nbk);
        }
      }
      phase ^= 1;
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =====================================
    // bf16 cache: kind::f16 products of bf16 operands. FP8 cache: kind::f8f6f4
    // products of E4M3 operands straight from the ring (K, V), with q and P
    // each given as an exact E4M3 pair hi + lo (two products per step).
    constexpr uint32_t idesc_qk = idesc_f16(128, 64, kFp8 ? 0 : 1, 0, 0);
    // PV: N = 128, the products with P's hi and lo parts side by side
    constexpr uint32_t idesc_pv = idesc_f16(128, 128, kFp8 ? 0 : 1, 1, 1);
    constexpr uint32_t kIPT = kItemsPerTensor<kFp8>;
    const uint32_t q_base = smem_u32(sQ);
    const uint32_t ring_base = smem_u32(sRing);
    const uint32_t p_base = smem_u32(sP);
    TileStream qs;
    qs.init(p, c.b_start, c.off_start, c.tiles, c.t0, c.L_start);
    uint32_t nq = 0;
    bool ok = true;
    // Ring items, in the producer's order K0 | K1 V0 | K2 V1 | ... | V(T-1),
    // kIPT per tensor: the first item of K(j) and of V(j) (the CTA's j-th tile).
    auto k_item = [](uint32_t j) -> uint32_t { return j == 0 ? 0u : (2u * j - 1u) * kIPT; };
    auto v_first = [](uint32_t j, bool cta_last) -> uint32_t {
      return (cta_last ? 2u * j + 1u : 2u * j + 2u) * kIPT;
    };
    // every lane tests (each acquires on success); the warp agrees
    auto items_ready = [&](uint32_t first) -> bool {
      bool r = true;
      for (uint32_t u = 0; u < kIPT; ++u)
        r = r && mbar_test_wait(&c.slot_full[(first + u) % kS], par((first + u) / kS));
      return __all_sync(0xffffffffu, r);
    };

    auto issue_pv = [&](const TileInfo& t, uint32_t j) {
      const uint32_t lo = v_first(j, t.cta_last);
      tc_fence_after();
      if (lane == 0) MFA_TR(3, j);
      // the whole warp issues (one elected lane; see mma_f16_ss_warp)
      if (kFp8) {
        // V slot: head dims 0-127 | 128-255, each 128 token rows of 128 B
        // (MN-major A); P: 128 token rows of hi (64 B) and lo (64 B) as two
        // 64-byte-swizzled blocks 8 KB apart (one N = 128 MN-major B)
        const uint32_t v = ring_base + (lo % kS) * kSlotBytes;
#pragma unroll
        for (int kk = 0; kk < kTile / 32; ++kk)
#pragma unroll
          for (int r = 0; r < 2; ++r)
            mma_f8_ss_warp(tmem + o_pv<kFp8>(t.seg, r),
                           sw128_desc(v + r * (kSlotBytes / 2) + kk * 4096, kSlotBytes / 2, 1024),
                           sw64_desc(p_base + kk * 2048, kPBytes / 2, 512), idesc_pv,
                           (t.seg_first && kk == 0) ? 0u : 1u);
        mma_commit_warp(&c.slot_empty[lo % kS]);
      } else {
        // V: two slots (head dims 0-127 | 128-255), each 128 token rows of
        // 64-dim chunks (MN-major A); P: 128 token rows of the hi and the lo
        // block (128 B each), 16 KB apart (one N = 128 MN-major B)
        const uint32_t hi = lo + 1;
        const uint32_t v_lo = ring_base + (lo % kS) * kSlotBytes;
        const uint32_t v_hi = ring_base + (hi % kS) * kSlotBytes;
        // the two head-dim halves accumulate into different columns: issue
        // them alternately, so consecutive products do not wait on each other
#pragma unroll
        for (int s = 0; s < kTile / 16; ++s) {
          mma_f16_ss_warp(tmem + o_pv<kFp8>(t.seg, 0),
                          sw128_desc(v_lo + s * 2048, kSlotBytes / 2, 1024),
                          sw128_desc(p_base + s * 2048, kPBlock, 1024), idesc_pv,
                          (t.seg_first && s == 0) ? 0u : 1u);
          mma_f16_ss_warp(tmem + o_pv<kFp8>(t.seg, 1),
                          sw128_desc(v_hi + s * 2048, kSlotBytes / 2, 1024),
                          sw128_desc(p_base + s * 2048, kPBlock, 1024), idesc_pv,
                          (t.seg_first && s == 0) ? 0u : 1u);
        }
        mma_commit_warp(&c.slot_empty[lo % kS]);
        mma_commit_warp(&c.slot_empty[hi % kS]);
      }
      mma_commit_warp(&c.o_full);
    };

    auto issue_qk = [&](const TileInfo& t, uint32_t j, uint32_t qbuf) {
      const uint32_t lo = k_item(j);
      tc_fence_after();
      if (lane == 0) MFA_TR(2, j);
      const uint32_t d_s = tmem + s_cols<kFp8>(j);
      if (kFp8) {
        // K slot: head dims 0-127 | 128-255 (128 token rows of 128 B, K-major);
        // q: per dims half, the 64 hi rows then the 64 lo rows (128 B each,
        // K-major): two N = 64 operands, both accumulated into S
        const uint32_t k = ring_base + (lo % kS) * kSlotBytes;
        const uint32_t qb = q_base + qbuf * kQBytes;
#pragma unroll
        for (int kk = 0; kk < kDim / 32; ++kk) {
          const uint32_t off = (kk >> 2) * (kSlotBytes / 2) + (kk & 3) * 32;
#pragma unroll
          for (int part = 0; part < 2; ++part)
            mma_f8_ss_warp(d_s, sw128_desc(k + off, 16, 1024),
                           sw128_desc(qb + off + part * (kQBytes / 4), 16, 1024), idesc_qk,
                           (kk > 0 || part > 0) ? 1u : 0u);
        }
        mma_commit_warp(&c.slot_empty[lo % kS]);
      } else {
        const uint32_t hi = lo + 1;
        const uint32_t k_lo = ring_base + (lo % kS) * kSlotBytes;
        const uint32_t k_hi = ring_base + (hi % kS) * kSlotBytes;
#pragma unroll
        for (int s = 0; s < kDim / 16; ++s) {
          const uint32_t a_addr = (s < 8 ? k_lo : k_hi) + ((s >> 2) & 1) * (kSlotBytes / 2) +
                                  (s & 3) * 32;
          const uint32_t b_addr = q_base + (s >> 2) * 8192 + (s & 3) * 32;
          mma_f16_ss_warp(d_s, sw128_desc(a_addr, 16, 1024), sw128_desc(b_addr, 16, 1024),
                          idesc_qk, s > 0 ? 1u : 0u);
        }
        mma_commit_warp(&c.slot_empty[lo % kS]);
        mma_commit_warp(&c.slot_empty[hi % kS]);
      }
      mma_commit_warp(&c.s_full[j & 1]);
      if (t.seg_last) mma_commit_warp(&c.q_empty[qbuf]);
    };

    // Each round issues the scores of tile g and the PV product of tile g - 1,
    // in that order. With an FP8 cache, while both are pending, the warp polls
    // both and issues whichever has its inputs first, the scores preferred (the
    // softmax needs S(g) before it needs PV(g - 1) done), so the PV product does
    // not wait behind a late K tile; the one left is then awaited as before.
    // (Measured: FP8 workload 72.8 -> 71.8 us; with a bf16 cache the polling
    // warp slowed the HBM-bound pipeline, 54.4 -> 57.6 us, so it keeps the
    // plain order.) Every wait is bounded.
    auto wait_items = [&](uint32_t first) -> bool {
      for (uint32_t u = 0; u < kIPT; ++u)
        if (!mbar_wait_warp(&c.slot_full[(first + u) % kS], par((first + u) / kS), abort_flag))
          return false;
      return true;
    };
    TileInfo cur, prev;
    uint32_t g = 0;
    uint32_t qbuf = 0;  // q buffer of the current segment
    bool have_cur = qs.next(cur), pending_pv = false;
    while (ok && (have_cur || pending_pv)) {
      bool need_qk = have_cur, need_pv = pending_pv;
      if (have_cur && cur.seg_first) qbuf = kTwoQ ? (nq & 1u) : 0u;
      uint64_t* qbar = kFp8 ? &c.q_conv[qbuf] : &c.q_full[0];
      const uint32_t qpar = kTwoQ ? par(nq >> 1) : par(nq);
      if (kFp8 && need_qk && need_pv) {
        const uint64_t t0 = global_timer_ns();
        for (uint32_t spin = 1;; ++spin) {
          if ((!cur.seg_first || __all_sync(0xffffffffu, mbar_test_wait(qbar, qpar))) &&
              (g < 2 || __all_sync(0xffffffffu,
                                   mbar_test_wait(&c.s_empty[g & 1], par((g >> 1) - 1)))) &&
              items_ready(k_item(g))) {
            issue_qk(cur, g, qbuf);
            need_qk = false;
            break;
          }
          if (__all_sync(0xffffffffu, mbar_test_wait(&c.p_full, par(g - 1))) &&
              items_ready(v_first(g - 1, prev.cta_last))) {
            issue_pv(prev, g - 1);
            need_pv = false;
            break;
          }
          if ((spin & 255u) == 0) {
            bool stop = *abort_flag != 0;
            if (!stop && global_timer_ns() - t0 > kWaitLimitNs) {
              if (lane == 0) {
                record_error(6 /* MFA_ERR_TIMEOUT */);
                *abort_flag = 1;
              }
              stop = true;
            }
            if (__any_sync(0xffffffffu, stop)) {
              ok = false;
              break;
            }
          }
        }
      }
#ifdef MFA_TRACE
      if (g == 0 && have_cur) {  // first tile: when K(0), then q, is in place
        wait_items(k_item(0));
        if (lane == 0) MFA_TR(12, 2);
        mbar_wait_warp(qbar, qpar, abort_flag);
        if (lane == 0) MFA_TR(12, 1);
      }
#endif
      if (ok && need_qk) {
        ok = (!cur.seg_first || mbar_wait_warp(qbar, qpar, abort_flag)) &&
             (g < 2 || mbar_wait_warp(&c.s_empty[g & 1], par((g >> 1) - 1), abort_flag)) &&
             wait_items(k_item(g));
        if (ok) issue_qk(cur, g, qbuf);
      }
      if (ok && need_pv) {
        ok = mbar_wait_warp(&c.p_full, par(g - 1), abort_flag) &&
             wait_items(v_first(g - 1, prev.cta_last));
        if (ok) issue_pv(prev, g - 1);
      }
      if (!ok) break;
      if (have_cur) {
        if (cur.seg_first) ++nq;
        prev = cur;
        ++g;
        pending_pv = true;  // PV of the tile just scored
        have_cur = qs.next(cur);
      } else {
        pending_pv = false;  // this round issued the last tile's PV
      }
    }
    if (!ok && lane == 0) {
      // drain: wait (bounded, ignoring the abort flag) for issued MMAs
      mma_commit(&c.drain);
      const uint64_t t0 = global_timer_ns();
      while (!mbar_try_wait(&c.drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ======================= q producer (FP8 cache: and publisher) ==========
    // q of segment k goes to buffer k & 1 (FP8: the next segment's q is loaded
    // and converted while this one runs) or the only buffer (bf16). With an
    // FP8 cache this warp also publishes each finished segment (warp 3
    // converts there), one segment behind: segment k - 1 after q of segment k
    // is on its way, since k - 1's last PV is issued after k's first QK.
    const uint64_t policy = l2_policy_evict_last();
    if (p.q_after_proj) griddep_wait();  // q is the projection grid's output
    TileStream qs, ahead;
    qs.init(p, c.b_start, c.off_start, c.tiles, c.t0, c.L_start);
    ahead.init(p, c.b_start, c.off_start, c.tiles, c.t0, c.L_start);
    TileInfo t, ta, last;
    bool more_ahead = ahead.next(ta);  // stays one segment ahead of qs
    bool have_last = false, ok = true;
    uint32_t k = 0;
    while (ok && qs.next(t)) {
      if (t.seg_first) {
        const uint32_t b = kTwoQ ? (k & 1u) : 0u;
        if (!(ok = mbar_wait_warp(&c.q_empty[b], (kTwoQ ? par(k >> 1) : par(k)) ^ 1u, abort_flag))) break;
        if (lane == 0) {
          if (!kFp8 && p.gqa) {
            // boxes of 64 dims x 32 heads: group g's dims half r into q region
            // 2 g + r, rows 32 g .. 32 g + 31
            mbar_arrive_expect_tx(&c.q_full[b], kQBytes / 2);
            for (int r = 0; r < 4; ++r)
              tma_load_3d(sQ + b * kQBytes + r * 8192 + (r >> 1) * 4096, &tm_q, &c.q_full[b],
                          (r & 1) * 64, (r >> 1) * 32, t.b, policy);
          } else {
            mbar_arrive_expect_tx(&c.q_full[b], kQBytes);
            for (int r = 0; r < 4; ++r)
              tma_load_3d(sQ + b * kQBytes + r * 8192, &tm_q, &c.q_full[b], r * 64, 0, t.b, policy);
          }
          MFA_TR(12, 0);
        }
        // pull the next segment's q rows into L2 while this segment runs
        while (more_ahead && (ta.b == t.b || !ta.seg_first)) more_ahead = ahead.next(ta);
        if (more_ahead && lane == 0) {
          if (!kFp8 && p.gqa) {
            for (int r = 0; r < 4; ++r) tma_prefetch_3d(&tm_q, (r & 1) * 64, (r >> 1) * 32, ta.b);
          } else {
            for (int r = 0; r < 4; ++r) tma_prefetch_3d(&tm_q, r * 64, 0, ta.b);
          }
        }
        __syncwarp();
        ++k;
        if (kFp8 && have_last && last.slot >= 0) {
          if (!(ok = __all_sync(0xffffffffu,
                                wait_count(&c.seg_arrivals, 4u * kWG * (k - 1), abort_flag))))
            break;
          if (lane == 0) publish_segment(p, last);
          __syncwarp();
        }
        have_last = false;
      }
      if (kFp8 && t.seg_last) {
        last = t;
        have_last = true;
      }
    }
    if (kFp8 && ok && have_last && last.slot >= 0 &&
        __all_sync(0xffffffffu, wait_count(&c.seg_arrivals, 4u * kWG * k, abort_flag))) {
      if (lane == 0) publish_segment(p, last);
      __syncwarp();
    }
  } else if (warp == 3) {
    // ======================= FP8 converter ==================================
    // Follows the MMA's consumption order: q at each segment start, then K of
    // tile g and V of tile g-1, each half-tile expanded in place to f16.
    if (kFp8) {
      // ======================= q to E4M3 (FP8 cache) ======================
      // Per segment, after q has landed: q becomes its exact E4M3 pair (see
      // q_to_e4m3) in place; the score scale 1/s goes to the softmax warps
      // through a four-entry ring (this warp runs at most two segments ahead
      // of them: q of the next segment waits for the current one's last QK).
      TileStream cs;
      cs.init(p, c.b_start, c.off_start, c.tiles, c.t0, c.L_start);
      TileInfo t;
      uint32_t nq = 0;
      while (cs.next(t)) {
        if (!t.seg_first) continue;
        const uint32_t b = kTwoQ ? (nq & 1u) : 0u;  // q buffer of segment nq
        const bool got = mbar_wait_warp(&c.q_full[b], kTwoQ ? par(nq >> 1) : par(nq), abort_flag);
        // the first segment with the softmax warps (they call the same function)
        const float inv_s = nq == 0 ? q_to_e4m3_group(smem_u32(sQ), tid - 96, got, true, c.qmax)
                            : got   ? q_to_e4m3(smem_u32(sQ + b * kQBytes), lane)
                                    : 0.f;
        if (!got) break;
        if (lane == 0) c.qinv[nq & 3] = inv_s;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&c.q_conv[b]);
          smem_add_release(&c.q_ready, 1u);
        }
        ++nq;
      }
    } else {
      // ======================= segment publisher (bf16 cache) ==============
      // After the softmax warps have written a segment's output or partial,
      // makes it visible device-wide and tells the combine kernel.
      TileStream ns;
      ns.init(p, c.b_start, c.off_start, c.tiles, c.t0, c.L_start);
      TileInfo t;
      unsigned k = 0;
      while (ns.next(t)) {
        if (!t.seg_last) continue;
        ++k;
        if (t.slot < 0) continue;  // the output itself: nothing to publish
        if (!__all_sync(0xffffffffu, wait_count(&c.seg_arrivals, 4u * kWG * k, abort_flag))) break;
        if (lane == 0) publish_segment(p, t);
        __syncwarp();
      }
    }
  } else if (warp >= 4) {
    // ======================= softmax + epilogue =============================
    const int wg = (warp - 4) >> 2;   // heads [kWGHeads wg, kWGHeads (wg + 1))
    const int sub = warp & 3;         // TMEM sub-partition of this warp
    const int row = sub * 32 + lane;  // token row in S^T / head-dim row in O^T
    const int hbase = wg * kWGHeads;
    // per-head values (running maximum, row sums, output scale) live in lane
    // hl (16-head warpgroups: lanes l and l + 16 both hold head l)
    const int hl = lane & (kWGHeads - 1);
    const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
    TileStream ts;
    ts.init(p, c.b_start, c.off_start, c.tiles, c.t0, c.L_start);
    if (kFp8) {
      // the first segment's q conversion, with warp 3 (which publishes it)
      TileStream first = ts;
      TileInfo tf;
      if (first.next(tf)) {
        const bool got = mbar_wait_warp(&c.q_full[0], 0u, abort_flag);
        q_to_e4m3_group(smem_u32(sQ), tid - 96, got, false, c.qmax);
      }
    }
    TileInfo t;
    uint32_t g = 0, nseg = 0;
    float m_run = -INFINITY;  // running max in use (log2 units), head hbase + hl
    float l_part[kWGHeads];
#pragma unroll
    for (int h = 0; h < kWGHeads; ++h) l_part[h] = 0.f;
    const float sl2 = p.score_log2;
    float ev = 0.f;  // output scale of the pending segment, head hbase + hl

    // Reads a finished segment's O (its own TMEM pair) and writes this warp's
    // share: the normalised output, or the partial of a split sequence. Then
    // hands the segment to its publisher: warp 3 for a bf16 cache (idle
    // there), so these warps go on without waiting for their stores to drain;
    // with an FP8 cache (warp 3 converts) every warp arrives itself.
    TileInfo pend;
    bool have_pending = false;
    uint32_t pend_g = 0;  // tile counter of the pending segment's last tile
    auto write_segment = [&](const TileInfo& pt, bool add_lo) {
      segment_out<kFp8>(p.ws_o, p.out, p.out_f32, p.out_sb, p.out_sh, pt.slot, pt.b,
                        tmem + lane_addr + hbase, o_hi<kFp8>(pt.seg, 0), o_hi<kFp8>(pt.seg, 1),
                        o_lo<kFp8>(pt.seg, 0), o_lo<kFp8>(pt.seg, 1), add_lo, row, hbase,
                        ev, kFp8 ? 0 : p.gqa);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) smem_add_release(&c.seg_arrivals, 1u);
      if (warp == 4 && lane == 0) MFA_TR(8, pend_g);
    };

    float sl2_seg = sl2;  // score scale of the current segment
    while (ts.next(t)) {
      if (t.seg_first) {
        m_run = -INFINITY;  // (l_part is zero at every segment start)
        if (kFp8) {
          // q of this segment entered the products as q * s: scale by 1/s
          if (!__all_sync(0xffffffffu, wait_count(&c.q_ready, t.seg + 1, abort_flag))) break;
          sl2_seg = sl2 * c.qinv[t.seg & 3];
        }
      }
      // ---- scores of this tile (this warpgroup's 32 heads) ---------------
      if (!mbar_wait_warp(&c.s_full[g & 1], par(g >> 1), abort_flag)) break;
      if (warp == 4 && lane == 0) MFA_TR(4, g);
      tc_fence_after();
      // scaled scores (log2 units); the maximum's own term is then exactly 0
      float s[kWGHeads];
      {
        uint32_t r[kWGHeads];
        tmem_ldw<kWGHeads>(tmem + lane_addr + s_cols<kFp8>(g) + hbase, r);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < kWGHeads; ++h) s[h] = __uint_as_float(r[h]) * sl2_seg;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.s_empty[g & 1]);

      const int valid = min(kTile, t.L - t.tile * kTile);
      const bool row_ok = row < valid;
      if (valid < kTile && !row_ok) {  // rows past the end: no weight
#pragma unroll
        for (int h = 0; h < kWGHeads; ++h) s[h] = -INFINITY;
      }

      // ---- per-head maximum over the tile's 128 rows --------------------
      {
        // per head, the maximum over this warp's 32 rows (every lane gets all
        // 32); lane 0 hands them to the exchange
        float r[kWGHeads];
#pragma unroll
        for (int h = 0; h < kWGHeads; ++h) r[h] = warp_max_f32(s[h]);
        if (lane == 0) {
          const uint32_t dst = smem_u32(&c.red[g & 1][wg][sub][0]);
#pragma unroll
          for (int q = 0; q < kWGHeads / 4; ++q)
            st_shared_v4(dst + 16 * q, __float_as_uint(r[4 * q]), __float_as_uint(r[4 * q + 1]),
                         __float_as_uint(r[4 * q + 2]), __float_as_uint(r[4 * q + 3]));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.red_full[wg][g & 1]);
      if (!mbar_wait_warp(&c.red_full[wg][g & 1], par(g >> 1), abort_flag)) break;
      if (warp == 4 && lane == 0) MFA_TR(5, g);
      const float tmax = fmaxf(fmaxf(c.red[g & 1][wg][0][hl], c.red[g & 1][wg][1][hl]),
                               fmaxf(c.red[g & 1][wg][2][hl], c.red[g & 1][wg][3][hl]));
      // lazy rescaling: move the reference max only when the tile's max
      // exceeds it by more than the threshold (exact: the factor cancels)
      float corr = 1.f;
      if (tmax > m_run + kRescaleThreshold) {
        corr = ex2_approx(m_run - tmax);
        m_run = tmax;
      }
      const bool rescale = __any_sync(0xffffffffu, corr != 1.f);
      float* mv = c.mv[g & 1][wg];  // every warp of the warpgroup stores the same values
      mv[hl] = m_run;
      __syncwarp();

      // ---- probabilities, row sums ---------------------------------------
      if (rescale) {  // (rare) the row sums move to the new reference first
#pragma unroll
        for (int h = 0; h < kWGHeads; ++h) l_part[h] *= __shfl_sync(0xffffffffu, corr, h);
      }
      // packed P: bf16 hi parts in pk, lo parts (p - hi, rounded) in pl; FP8
      // E4M3 hi bytes in pk[0..7], lo bytes in pk[8..15]
      uint32_t pk[kWGHeads / 2];
      uint32_t pl[kFp8 ? 1 : kWGHeads / 2];
#pragma unroll
      for (int h = 0; h < kWGHeads; h += 4) {
        const float4 m4 = *reinterpret_cast<const float4*>(&mv[h]);
        const float p0 = ex2_approx(s[h] - m4.x);
        const float p1 = ex2_approx(s[h + 1] - m4.y);
        const float p2 = ex2_approx(s[h + 2] - m4.z);
        const float p3 = ex2_approx(s[h + 3] - m4.w);
        l_part[h] += p0;
        l_part[h + 1] += p1;
        l_part[h + 2] += p2;
        l_part[h + 3] += p3;
        if (kFp8) {
          // E4M3 pairs: hi bytes of heads h..h+3 in pk[h / 4], lo bytes in
          // pk[kWGHeads / 4 + h / 4]
          const uint32_t a = split_e4m3x2(p0, p1), b = split_e4m3x2(p2, p3);
          pk[h / 4] = (a & 0xFFFFu) | (b << 16);
          pk[kWGHeads / 4 + h / 4] = (a >> 16) | (b & 0xFFFF0000u);
        } else {
          // p = hi + lo to ~16 significant bits: the PV product's error is then
          // far below that of a single bf16 rounding (2^-9 relative)
          const uint32_t a = pack_bf16x2(p0, p1), b = pack_bf16x2(p2, p3);
          pk[h / 2] = a;
          pk[h / 2 + 1] = b;
          pl[h / 2] = pack_bf16x2(p0 - __uint_as_float(a << 16), p1 - __uint_as_float(a & 0xFFFF0000u));
          pl[h / 2 + 1] =
              pack_bf16x2(p2 - __uint_as_float(b << 16), p3 - __uint_as_float(b & 0xFFFF0000u));
        }
      }

      // ---- P buffer and O are free once the previous tile's PV completed --
      if (warp == 4 && lane == 0) MFA_TR(6, g);
      if (g >= 1 && !mbar_wait_warp(&c.o_full, par(g - 1), abort_flag)) break;
      tc_fence_after();
      if (rescale && !t.seg_first) {
        constexpr int kChunks = kWGHeads / 16;  // 16-column chunks of this warp's heads
#pragma unroll 1
        for (int q4 = 0; q4 < 4 * kChunks; ++q4) {  // (hi, lo) x halves x chunks
          uint32_t r[16];
          const int cb = (q4 % kChunks) * 16, half = (q4 / kChunks) & 1;
          const uint32_t a =
              tmem + lane_addr +
              ((q4 / (2 * kChunks)) ? o_lo<kFp8>(t.seg, half) : o_hi<kFp8>(t.seg, half)) + hbase +
              cb;
          tmem_ld16(a, r);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            r[j] = __float_as_uint(__uint_as_float(r[j]) * __shfl_sync(0xffffffffu, corr, cb + j));
          tmem_st16(a, r);
        }
        tmem_wait_st();
      }
      if (!kFp8 && have_pending) {
        // first tile of a new segment (bf16): the previous segment's last PV
        // has completed (the wait above); add its lo part into its hi columns
        // before this tile's PV overwrites the shared lo columns
        constexpr int kChunks = kWGHeads / 16;
#pragma unroll 1
        for (int q4 = 0; q4 < 2 * kChunks; ++q4) {  // halves x 16-column chunks
          uint32_t a[16], b[16];
          const int cb = (q4 % kChunks) * 16, half = q4 / kChunks;
          const uint32_t ha = tmem + lane_addr + o_hi<kFp8>(pend.seg, half) + hbase + cb;
          tmem_ld16(ha, a);
          tmem_ld16(tmem + lane_addr + o_lo<kFp8>(pend.seg, half) + hbase + cb, b);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            a[j] = __float_as_uint(__uint_as_float(a[j]) + __uint_as_float(b[j]));
          tmem_st16(ha, a);
        }
        tmem_wait_st();
      }
      if (kFp8) {
        // P hi | lo: 128 token rows of 64 heads (64 B, 64-byte swizzle); this
        // warpgroup's heads are the row's 16-byte chunks kC wg .. kC wg + kC - 1
        constexpr int kC = kWGHeads / 16;
        const uint32_t rowaddr = smem_u32(sP) + row * 64;
        const int sw = (row >> 1) & 3;
#pragma unroll
        for (int part = 0; part < 2; ++part)
#pragma unroll
          for (int ch = 0; ch < kC; ++ch)
            st_shared_v4(rowaddr + part * (kPBytes / 2) + (((kC * wg + ch) ^ sw) << 4),
                         pk[(kWGHeads / 4) * part + 4 * ch], pk[(kWGHeads / 4) * part + 4 * ch + 1],
                         pk[(kWGHeads / 4) * part + 4 * ch + 2],
                         pk[(kWGHeads / 4) * part + 4 * ch + 3]);
      } else {
        // P hi and lo blocks: 128 token rows of 64 heads (128 B, 128-byte
        // swizzle); this warpgroup's heads are 16-byte chunks kC wg ..
        // kC wg + kC - 1. Even segments put the hi block first, odd ones the lo
        // block (the TMEM column map above).
        constexpr int kC = kWGHeads / 8;
        const uint32_t rowaddr = smem_u32(sP) + row * 128;
        const uint32_t hi_off = (t.seg & 1) ? kPBlock : 0u;
#pragma unroll
        for (int ch = 0; ch < kC; ++ch) {
          const uint32_t a = rowaddr + (((kC * wg + ch) ^ (row & 7)) << 4);
          st_shared_v4(a + hi_off, pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
          st_shared_v4(a + (kPBlock - hi_off), pl[4 * ch], pl[4 * ch + 1], pl[4 * ch + 2],
                       pl[4 * ch + 3]);
        }
      }
      // rows past the sequence end: zero the V rows so 0 * (stale or NaN) never
      // reaches the accumulator. bf16 (two warpgroups): warpgroup w takes the
      // item of head dims 128 w .. 128 w + 127 (two 64-dim regions). FP8: the
      // tensor's one item (two 16 KB halves of 128-byte rows); warpgroup w
      // takes half w & 1, bytes kRowPart (w >> 1) .. + kRowPart - 1 of each row.
      if (valid < kTile) {
        constexpr int kRowPart = kFp8 ? 256 / kWG : 128;  // bytes of a 128-byte row
        const uint32_t it = v_item<kFp8>(g, t.cta_last) + (kFp8 ? 0 : wg);
        if (!mbar_wait_warp(&c.slot_full[it % kS], par(it / kS), abort_flag)) break;
        if (!row_ok) {
          const uint32_t base =
              smem_u32(sRing) + (it % kS) * kSlotBytes + row * 128 +
              (kFp8 ? (wg & 1) * (kSlotBytes / 2) + (wg >> 1) * kRowPart : 0);
#pragma unroll
          for (int r = 0; r < (kFp8 ? 1 : 2); ++r)
#pragma unroll
            for (int ch = 0; ch < kRowPart / 16; ++ch)
              st_shared_v4(base + r * (kSlotBytes / 2) + ch * 16, 0u, 0u, 0u, 0u);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.p_full);
      if (warp == 4 && lane == 0) MFA_TR(7, g);

      // ---- output of the previous segment, deferred to here ---------------
      // Its last PV completed before this tile's P went out (the o_full wait
      // above) and the MMA now accumulates into the other O pair, so the
      // read-out overlaps this tile's PV and the next tile's QK. (An FP8
      // segment is read out at its end or after the loop, never here: the
      // condition keeps this copy of the read-out out of the FP8 loop's code.)
      if (!kFp8 && have_pending) {
        write_segment(pend, false);  // its lo part is in its hi columns now
        have_pending = false;
      }

      // ---- end of a segment: row sums and log-sum-exp ---------------------
      if (t.seg_last) {
        // the row sums travel through this tile's maxima buffer, once every
        // warp of the warpgroup has read its maxima (l_pre); it is next
        // written two tiles on, after every warp has passed the next tile's
        // maximum exchange (so after the reads below)
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.l_pre[wg]);
        if (!mbar_wait_warp(&c.l_pre[wg], par(nseg), abort_flag)) break;
        float* lred = &c.red[g & 1][wg][0][0];
        {
          float v[kWGHeads];
#pragma unroll
          for (int h = 0; h < kWGHeads; ++h) v[h] = l_part[h];
          const float rs = reduce_scatter<false>(v, lane);
          if (kWGHeads == 32)
            lred[sub * kWGHeads + lane] = rs;
          else if ((lane & 1) == 0)
            lred[sub * kWGHeads + (lane >> 1)] = rs;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.l_full[wg]);
        if (!mbar_wait_warp(&c.l_full[wg], par(nseg), abort_flag)) break;
        const float l = lred[hl] + lred[kWGHeads + hl] + lred[2 * kWGHeads + hl] +
                        lred[3 * kWGHeads + hl];
        // the next tile starts a new segment: the row sums restart from zero
#pragma unroll
        for (int h = 0; h < kWGHeads; ++h) l_part[h] = 0.f;
        const float lse = (m_run + lg2_approx(l)) * kLn2;  // head hbase + hl
        ev = p.out_scale / l;
        if (sub == 0 && lane < kWGHeads) {
          if (t.slot >= 0)
            p.ws_lse[static_cast<int64_t>(t.slot) * kHeads + hbase + lane] = lse;
          else if (p.lse_out)
            p.lse_out[t.b * p.lse_sb + hbase + lane] = lse;
        }
        __syncwarp();
        ++nseg;
        pend = t;
        pend_g = g;
        have_pending = true;
        if (kFp8 && !t.cta_last) {
          // single O buffer: read out now, before the next segment's first PV
          if (!mbar_wait_warp(&c.o_full, par(g), abort_flag)) break;
          tc_fence_after();
          write_segment(pend, true);
          have_pending = false;
        }
      }
      ++g;
    }
    // the CTA's last segment: after its last PV
    if (have_pending && !*abort_flag && mbar_wait_warp(&c.o_full, par(g - 1), abort_flag)) {
      tc_fence_after();
      write_segment(pend, true);
    }
  }

  // ---- teardown ------------------------------------------------------------
  if (tid == 0) MFA_TR(11, 0);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
#ifdef MFA_TRACE
  if (tid == 0) {
    MFA_GT(0, blockIdx.x, 2, gt_call);
    if (blockIdx.x < kGtCtas) g_mfa_cnt[blockIdx.x] = gt_call + 1;
  }
#endif
}

// ===========================================================================
// Split merge (Flash-Decoding's log-sum-exp combine) and empty sequences.
// CTA (b, q): sequence b, heads 16q..16q+15; thread = head-dim index.
//   lse* = max_s lse_s,  w_s = exp(lse_s - lse*),
//   out = sum_s w_s O_s / sum_s w_s,   lse = lse* + log(sum_s w_s)
// over the sequence's partials in plan order.
//
// The kernel starts while the attention kernel still runs (on SMs it has
// left), once every attention CTA has written its plan words and cleared its
// slot flags. A CTA derives its sequence's partial slots from the plan, waits
// (bounded) for their flags and merges, so merges overlap the attention
// kernel's last tiles; a sequence that one segment covers was finished by the
// attention kernel itself. One CTA waits for the attention grid to complete at
// its end, so a call is over when this kernel is.
// ===========================================================================
// kMinBlocks blocks per SM: 2 (128 registers, four partials per round trip)
// or, for batches whose blocks would not all fit at two per SM, 4 (64
// registers, two partials per round trip), so that a block waiting for a late
// sequence does not keep a block of a finished one from starting.
// (Measured: E4M3 batch 128, 71.3 -> 70.5 us with 4; bf16 batch 64, whose 256
// blocks fit at 2 per SM, 54.3 -> 55.9 us with 4.)
template <int kMinBlocks>
__global__ void __launch_bounds__(kDim, kMinBlocks) mfa_combine_kernel(const DecodeParams p) {
#ifdef MFA_TRACE
  const unsigned long long gt_start = global_timer_ns();
  const int cta_lin = blockIdx.x * gridDim.y + blockIdx.y;
#endif
  griddep_launch_dependents();
  const int b = blockIdx.x;
  const int q = blockIdx.y;
  const int h = q * kCombineHeads + (threadIdx.x >> 4);  // this thread's head
  const int d0 = (threadIdx.x & 15) * kCombineDims;       // and its 16 dims
  // the lengths are an input of the call: complete before the attention
  // kernel passed its own dependency wait, which precedes this kernel's start
  const int nt = tiles_of(valid_len(p, b));
#ifdef MFA_TRACE
  const int gt_call = cta_lin < kGtCtas ? *reinterpret_cast<volatile int*>(&g_mfa_cnt[kGtCtas + cta_lin]) : -1;
  if (threadIdx.x == 0) {
    MFA_GT(1, cta_lin, 1, gt_call);
    if (gt_call >= 0 && gt_call < kGtCalls && cta_lin < kGtCtas)
      g_mfa_gt[((gt_call * 2 + 1) * kGtCtas + cta_lin) * 3] = gt_start;
  }
  struct GtEnd {
    int call, cta;
    __device__ ~GtEnd() {
      __syncthreads();
      if (threadIdx.x == 0) {
        MFA_GT(1, cta, 2, call);
        if (cta < kGtCtas) g_mfa_cnt[kGtCtas + cta] = call + 1;
      }
    }
  } gt_end{gt_call, cta_lin};
#endif

  // grouped-query mode: 128 output dims per head (partials keep their 256-wide
  // rows, the group's values in the first 128)
  const bool dims_ok = !p.gqa || d0 < kDim / 2;
  if (nt == 0) {  // empty sequence: zeros, lse = -inf
    float v[kCombineDims];
#pragma unroll
    for (int j = 0; j < kCombineDims; ++j) v[j] = 0.f;
    if (dims_ok) store_out16(p, b, h, d0, v);
    if (p.lse_out && d0 == 0) p.lse_out[b * p.lse_sb + h] = -INFINITY;
  } else {
    const SplitList sl = split_list_of(p, b, nt);
    // a sequence spans at most grid + 1 CTAs (balanced) or num_splits units
    const int max_count = p.num_splits == 0 ? p.grid + 1 : p.num_splits;
    const int nslots = p.num_splits == 0 ? 2 * p.grid : p.batch * p.num_splits;
    const bool sane = sl.count >= 1 && sl.count <= max_count;
    if (!sane && threadIdx.x == 0) record_error(5 /* MFA_ERR_BAD_INDEX */);
    if (sane && sl.nonempty() > 1) {  // split: wait for every partial, then merge
      __shared__ int s_ok;
      if (threadIdx.x == 0) s_ok = 1;
      __syncthreads();
      for (int i = threadIdx.x; i < sl.count; i += blockDim.x) {
        const int slot = sl.slot(i);
        if (slot >= nslots) {
          record_error(5 /* MFA_ERR_BAD_INDEX */);
          s_ok = 0;
        } else if (slot >= 0 && !wait_flag(p.ws_flag + slot, p.wait_ns)) {
          s_ok = 0;
        }
      }
      __syncthreads();
      if (s_ok && dims_ok) merge_head_part<kMinBlocks == 4 ? 2 : 4>(p, b, sl, h, d0);
    }
  }
  // One block waits for the attention grid to complete, so this grid never
  // completes before it: a later kernel that waits for this one (the next
  // call) also waits for the attention kernel. The other blocks leave as soon
  // as their sequence is merged, so the blocks that did not fit beside the
  // attention CTAs (large batches) start without waiting for that grid's end.
  if (blockIdx.x == 0 && blockIdx.y == 0) griddep_wait();
}

// ===========================================================================
// host-side launch helper (called from mfa_api.cu)
// ===========================================================================
int decode_smem_bytes() {
  constexpr int a = SmemLayout<false>::kBytes, b = SmemLayout<true>::kBytes,
                c = SmemLayout<true, true>::kBytes;
  return a > b ? (a > c ? a : c) : (b > c ? b : c);
}

template <typename Kernel, typename... Args>
static cudaError_t launch_pdl(Kernel kernel, dim3 grid, dim3 block, size_t smem,
                              cudaStream_t stream, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

template <bool kPaged, bool kFp8, bool kOneQ>
static cudaError_t launch_attention(const CUtensorMap& tq, const CUtensorMap& tk,
                                    const CUtensorMap& tv, const DecodeParams& p,
                                    cudaStream_t stream) {
  static thread_local int configured_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (configured_dev != dev) {
    const cudaError_t err = cudaFuncSetAttribute(
        mfa_decode_kernel<kPaged, kFp8, kOneQ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
        SmemLayout<kFp8, kOneQ>::kBytes);
    if (err != cudaSuccess) return err;
    configured_dev = dev;
  }
  return launch_pdl(mfa_decode_kernel<kPaged, kFp8, kOneQ>, dim3(p.grid),
                    dim3(Geo<kFp8>::kThreads), SmemLayout<kFp8, kOneQ>::kBytes, stream, tq, tk,
                    tv, p);
}

// The combine variant for this batch (blocks per SM, above).
static bool combine_wide(const DecodeParams& p) {
  return static_cast<long long>(p.batch) * (kHeads / kCombineHeads) > 2LL * p.grid;
}

// The combine kernel alone, without programmatic launch (failure self-test).
cudaError_t launch_combine_only(const DecodeParams& p, cudaStream_t stream) {
  if (combine_wide(p))
    mfa_combine_kernel<4><<<dim3(p.batch, kHeads / kCombineHeads), dim3(kDim), 0, stream>>>(p);
  else
    mfa_combine_kernel<2><<<dim3(p.batch, kHeads / kCombineHeads), dim3(kDim), 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_decode(bool paged, bool fp8, const CUtensorMap& tq, const CUtensorMap& tk,
                          const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream) {
  cudaError_t err;
  // FP8 with at most one unit (so one segment) per CTA: one q buffer, a deeper ring
  const bool one_q =
      p.num_splits > 0 && static_cast<long long>(p.batch) * p.num_splits <= p.grid;
  if (fp8 && one_q)
    err = paged ? launch_attention<true, true, true>(tq, tk, tv, p, stream)
                : launch_attention<false, true, true>(tq, tk, tv, p, stream);
  else if (fp8)
    err = paged ? launch_attention<true, true, false>(tq, tk, tv, p, stream)
                : launch_attention<false, true, false>(tq, tk, tv, p, stream);
  else
    err = paged ? launch_attention<true, false, true>(tq, tk, tv, p, stream)
                : launch_attention<false, false, true>(tq, tk, tv, p, stream);
  if (err != cudaSuccess) return err;
  return combine_wide(p) ? launch_pdl(mfa_combine_kernel<4>, dim3(p.batch, kHeads / kCombineHeads),
                                      dim3(kDim), 0, stream, p)
                         : launch_pdl(mfa_combine_kernel<2>, dim3(p.batch, kHeads / kCombineHeads),
                                      dim3(kDim), 0, stream, p);
}

}  // namespace mfa
