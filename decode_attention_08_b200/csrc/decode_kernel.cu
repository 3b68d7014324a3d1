// decode_kernel.cu -- MFA decode attention on sm_100a (bf16 KV cache).
//
// Step-3 page, "Key points -> Architecture": the 64 query heads of a token all
// attend over ONE shared key head and ONE shared value head of dimension 256.
// Because every cached row is shared by all 64 heads, both products of the
// attention are dense contractions and run on the 5th-generation tensor core:
//
//   S^T[t, h] = sum_i K[t, i] * q[h, i]       M = 128 tokens, N = 64 heads, K = 256
//   O^T[i, h] += sum_t V[t, i] * P[h, t]      M = 128 dims (x2), N = 64 heads, K = 128 tokens
//
// Both are issued "swap-AB" (tokens / head dims on the MMA's M side) so every
// accumulator uses the M = 128 TMEM layout where TMEM lane = matrix row. The
// softmax is computed online over 128-token tiles (running max with lazy
// rescaling, running sum), so each K and V row is read from HBM exactly once.
//
// CTA = 8 warps, one CTA per SM (persistent):
//   warp 0  TMA producer for the K/V ring (5 slots x 32 KB)
//   warp 1  TMEM allocator + single-thread tcgen05.mma issuer
//   warp 2  TMA producer for q (one 32 KB load per sequence segment)
//   warp 3  idle
//   warps 4-7  softmax + epilogue (thread = one token row of S^T, then one
//              head-dim row of O^T)
//
// Work split (Flash-Decoding, cited on the DeepSeek-V4 page): the (sequence,
// 128-token tile) pairs of the whole batch are cut into `grid` contiguous,
// equal ranges ("balanced"), or every sequence into `num_splits` equal ranges.
// A range that covers a whole sequence writes the final output; otherwise it
// writes a normalised partial and its log-sum-exp, merged by mfa_combine_kernel.
// The plan depends only on seq_lens, num_splits and grid, never on whether the
// cache is paged, so paged and contiguous caches give bit-identical results.

#include "mfa_internal.h"
#include "sm100.cuh"

namespace mfa {

namespace {

// ---------------------------------------------------------------------------
// shared-memory control block
// ---------------------------------------------------------------------------
struct __align__(16) DecodeCtrl {
  uint64_t q_full, q_empty;
  uint64_t slot_full[kSlots], slot_empty[kSlots];
  uint64_t s_full[2], s_empty[2];
  uint64_t p_full, o_full;
  uint64_t red_full[2], l_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  int b_start, off_start, tiles;
  int scan_warp[8];
  float red[2][4][kHeads];   // per-warp tile maxima
  float mv[4][kHeads];       // per-warp copy of the running max in use
  float cv[4][kHeads];       // per-warp copy of the rescale factors
  float lred[4][kHeads];     // per-warp partial row sums (epilogue)
};

constexpr int kSmemQ = 0;
constexpr int kSmemRing = kSmemQ + kQBytes;
constexpr int kSmemP = kSmemRing + kSlots * kSlotBytes;
constexpr int kSmemCtrl = kSmemP + kPBytes;
constexpr int kSmemBytes = kSmemCtrl + static_cast<int>(sizeof(DecodeCtrl)) + 1024;

// TMEM column map.
constexpr uint32_t kColS = 0;      // two 64-column score buffers
constexpr uint32_t kColOlo = 128;  // O^T rows 0..127
constexpr uint32_t kColOhi = 192;  // O^T rows 128..255

__device__ __forceinline__ int tiles_of(int L) { return (L + kTile - 1) / kTile; }

__device__ __forceinline__ int valid_len(const DecodeParams& p, int b) {
  int L = __ldg(p.seq_lens + b);
  if (L < 0 || L > p.cap_tokens) {
    record_error(5 /* MFA_ERR_BAD_INDEX */);
    return 0;
  }
  return L;
}

// ---------------------------------------------------------------------------
// The per-CTA stream of tiles, walked independently (and identically) by each
// role.
// ---------------------------------------------------------------------------
struct TileInfo {
  int b;          // sequence
  int tile;       // tile index within the sequence
  int L;          // sequence length
  bool seg_first; // first tile of a segment (run of tiles of one sequence)
  bool seg_last;  // last tile of a segment
  bool cta_last;  // last tile this CTA processes
  int slot;       // partial slot of the segment, -1 when it covers the sequence
};

struct TileStream {
  const DecodeParams* p;
  int cta;
  // balanced plan
  int b, tile, L, nt, remaining, seg_lo, seg_hi, seg_ord;
  // fixed-splits plan
  int unit, unit_hi;

  __device__ void init(const DecodeParams& prm, int b_start, int off_start, int tiles) {
    p = &prm;
    cta = blockIdx.x;
    seg_ord = 0;
    if (prm.num_splits == 0) {
      remaining = tiles;
      if (remaining > 0) {
        b = b_start;
        L = valid_len(prm, b);
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
  __device__ void advance_unit() {
    const int s = p->num_splits;
    const int nunits = p->batch * s;
    for (unit += p->grid; unit < nunits; unit += p->grid) {
      b = unit / s;
      const int j = unit % s;
      L = valid_len(*p, b);
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
    const bool complete = (seg_lo == 0 && seg_hi == nt);
    if (p->num_splits == 0) {
      t.slot = complete ? -1 : (2 * cta + (seg_ord == 0 ? 0 : 1));
      ++tile;
      --remaining;
      t.cta_last = (remaining == 0);
      if (remaining > 0 && tile == nt) {
        do {
          ++b;
          L = valid_len(*p, b);
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
// Block-wide plan: total tiles, this CTA's tile range and its first sequence.
// CTA 0 also stores the per-sequence tile prefix for the combine kernel.
// ---------------------------------------------------------------------------
__device__ int block_inclusive_scan(int v, int* warp_sums) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  if (lane == 31) warp_sums[warp] = v;
  __syncthreads();
  int add = 0;
#pragma unroll
  for (int w = 0; w < kDecodeThreads / 32; ++w)
    if (w < warp) add += warp_sums[w];
  v += add;
  __syncthreads();
  return v;
}

__device__ void balanced_plan(const DecodeParams& p, DecodeCtrl& c) {
  const int tid = threadIdx.x;
  // pass 1: total number of tiles
  long long total = 0;
  for (int base = 0; base < p.batch; base += kDecodeThreads) {
    const int b = base + tid;
    const int n = (b < p.batch) ? tiles_of(valid_len(p, b)) : 0;
    const int incl = block_inclusive_scan(n, c.scan_warp);
    // the block's last thread holds the chunk total
    __shared__ int s_chunk;
    if (tid == kDecodeThreads - 1) s_chunk = incl;
    __syncthreads();
    total += s_chunk;
    __syncthreads();
  }
  const long long G = p.grid;
  const long long t0 = (static_cast<long long>(blockIdx.x) * total) / G;
  const long long t1 = (static_cast<long long>(blockIdx.x + 1) * total) / G;
  if (tid == 0) {
    c.tiles = static_cast<int>(t1 - t0);
    c.b_start = 0;
    c.off_start = 0;
  }
  // pass 2: locate tile t0; CTA 0 writes the prefix
  long long run = 0;
  for (int base = 0; base < p.batch; base += kDecodeThreads) {
    const int b = base + tid;
    const int n = (b < p.batch) ? tiles_of(valid_len(p, b)) : 0;
    const int incl = block_inclusive_scan(n, c.scan_warp);
    const long long excl = run + incl - n;
    if (b < p.batch) {
      if (blockIdx.x == 0 && p.ws_prefix) p.ws_prefix[b] = static_cast<int>(excl);
      if (n > 0 && excl <= t0 && t0 < excl + n) {
        c.b_start = b;
        c.off_start = static_cast<int>(t0 - excl);
      }
    }
    __shared__ int s_chunk2;
    if (tid == kDecodeThreads - 1) s_chunk2 = incl;
    __syncthreads();
    run += s_chunk2;
    __syncthreads();
  }
  if (blockIdx.x == 0 && tid == 0 && p.ws_prefix) p.ws_prefix[p.batch] = static_cast<int>(total);
  __syncthreads();
}

// ---------------------------------------------------------------------------
// warp-level "reduce-scatter" over the 32 rows a warp holds: on entry each lane
// has 64 per-head values of its own row; on exit lane l holds, in v[0] and v[1],
// the reduction over all 32 lanes for heads 2l and 2l+1.
// ---------------------------------------------------------------------------
template <bool kMax, int N, int MASK>
__device__ __forceinline__ void rs_step(float (&v)[64], int lane) {
  const bool upper = (lane & MASK) != 0;
#pragma unroll
  for (int i = 0; i < N / 2; ++i) {
    const float send = upper ? v[i] : v[i + N / 2];
    const float keep = upper ? v[i + N / 2] : v[i];
    const float recv = __shfl_xor_sync(0xffffffffu, send, MASK);
    v[i] = kMax ? fmaxf(keep, recv) : keep + recv;
  }
}

template <bool kMax>
__device__ __forceinline__ void reduce_scatter64(float (&v)[64], int lane) {
  rs_step<kMax, 64, 16>(v, lane);
  rs_step<kMax, 32, 8>(v, lane);
  rs_step<kMax, 16, 4>(v, lane);
  rs_step<kMax, 8, 2>(v, lane);
  rs_step<kMax, 4, 1>(v, lane);
}

// Softmax-side parity helper: phase parity of the u-th completion.
__device__ __forceinline__ uint32_t par(uint32_t u) { return u & 1u; }

// Index, in producer order, of the first (lo) ring item holding V of the CTA's
// j-th tile: items go K0 | K1 V0 | K2 V1 | ... | K(T-1) V(T-2) | V(T-1), two
// items (lo/hi head-dim halves) per tensor and tile.
__device__ __forceinline__ uint32_t v_item(uint32_t j, bool cta_last) {
  return cta_last ? 4u * j + 2u : 4u * j + 4u;
}

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: P entries stay <= 2^8

}  // namespace

// ===========================================================================
// the attention kernel
// ===========================================================================
template <bool kPaged>
__global__ void __launch_bounds__(kDecodeThreads, 1)
    mfa_decode_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem + kSmemQ;
  uint8_t* sRing = smem + kSmemRing;
  uint8_t* sP = smem + kSmemP;
  DecodeCtrl& c = *reinterpret_cast<DecodeCtrl*>(smem + kSmemCtrl);

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // ---- plan --------------------------------------------------------------
  if (p.num_splits == 0) {
    balanced_plan(p, c);
    if (c.tiles == 0) return;
  } else {
    if (static_cast<int>(blockIdx.x) >= p.batch * p.num_splits) return;
    if (tid == 0) {
      c.tiles = -1;
      c.b_start = 0;
      c.off_start = 0;
    }
  }

  // ---- setup -------------------------------------------------------------
  if (tid == 0) {
    mbar_init(&c.q_full, 1);
    mbar_init(&c.q_empty, 1);
    for (int i = 0; i < kSlots; ++i) {
      mbar_init(&c.slot_full[i], 1);
      mbar_init(&c.slot_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c.s_full[i], 1);
      mbar_init(&c.s_empty[i], 4);
      mbar_init(&c.red_full[i], 4);
    }
    mbar_init(&c.p_full, 4);
    mbar_init(&c.o_full, 1);
    mbar_init(&c.l_full, 4);
    mbar_init(&c.drain, 1);
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  volatile int* abort_flag = &c.abort_flag;
  const uint32_t tmem = c.tmem_base;

  if (warp == 0) {
    // ======================= K/V producer ===================================
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_first();
      TileStream ks, vs;
      ks.init(p, c.b_start, c.off_start, c.tiles);
      vs.init(p, c.b_start, c.off_start, c.tiles);
      uint32_t item = 0;
      bool ok = true;
      auto load = [&](const TileInfo& t, const CUtensorMap* map) -> bool {
        for (int half = 0; half < 2; ++half) {
          const uint32_t slot = item % kSlots;
          if (!mbar_wait(&c.slot_empty[slot], par(item / kSlots) ^ 1u, abort_flag)) return false;
          uint8_t* dst = sRing + slot * kSlotBytes;
          const int t0 = t.tile * kTile;
          if (!kPaged) {
            mbar_arrive_expect_tx(&c.slot_full[slot], kSlotBytes);
            for (int r = 0; r < 2; ++r)
              tma_load_3d(dst + r * (kSlotBytes / 2), map, &c.slot_full[slot],
                          (2 * half + r) * 64, t0, t.b, policy);
          } else {
            const int ps = p.page_size;
            const int rows = ps < kTile ? ps : kTile;
            const int nsub = kTile / rows;
            uint32_t bytes = 0;
            for (int j = 0; j < nsub; ++j)
              if (t0 + j * rows < t.L) bytes += rows * 128 * 2;
            mbar_arrive_expect_tx(&c.slot_full[slot], bytes);
            for (int j = 0; j < nsub; ++j) {
              const int tok = t0 + j * rows;
              if (tok >= t.L) break;
              const int lp = tok / ps;
              int phys = __ldg(p.page_table + static_cast<int64_t>(t.b) * p.pt_stride + lp);
              if (phys < 0 || phys >= p.num_pages) {
                record_error(5 /* MFA_ERR_BAD_INDEX */);
                phys = 0;
              }
              for (int r = 0; r < 2; ++r)
                tma_load_3d(dst + r * (kSlotBytes / 2) + j * rows * 128, map, &c.slot_full[slot],
                            (2 * half + r) * 64, tok % ps, phys, policy);
            }
          }
          ++item;
        }
        return true;
      };
      TileInfo kt, vt;
      bool more_k = ks.next(kt);
      bool first = true;
      while (ok) {
        if (more_k) ok = load(kt, &tm_k);
        if (ok && !first) {
          vs.next(vt);
          ok = load(vt, &tm_v);
        }
        if (!more_k) break;
        first = false;
        more_k = ks.next(kt);
      }
      (void)ok;
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =====================================
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_f16(128, 64, 1, 0, 0);
      constexpr uint32_t idesc_pv = idesc_f16(128, 64, 1, 1, 1);
      const uint32_t q_base = smem_u32(sQ);
      const uint32_t ring_base = smem_u32(sRing);
      const uint32_t p_base = smem_u32(sP);
      TileStream qs;
      qs.init(p, c.b_start, c.off_start, c.tiles);
      uint32_t item = 0, nq = 0;
      bool ok = true;

      auto issue_pv = [&](const TileInfo& t, uint32_t j) -> bool {
        if (!mbar_wait(&c.p_full, par(j), abort_flag)) return false;
        const uint32_t lo = item++, hi = item++;
        if (!mbar_wait(&c.slot_full[lo % kSlots], par(lo / kSlots), abort_flag)) return false;
        if (!mbar_wait(&c.slot_full[hi % kSlots], par(hi / kSlots), abort_flag)) return false;
        tc_fence_after();
        const uint32_t v_lo = ring_base + (lo % kSlots) * kSlotBytes;
        const uint32_t v_hi = ring_base + (hi % kSlots) * kSlotBytes;
#pragma unroll
        for (int s = 0; s < kTile / 16; ++s) {
          const uint64_t bdesc = sw128_desc(p_base + s * 2048, 8192, 1024);
          const uint32_t acc = (t.seg_first && s == 0) ? 0u : 1u;
          mma_f16_ss(tmem + kColOlo, sw128_desc(v_lo + s * 2048, kSlotBytes / 2, 1024), bdesc,
                     idesc_pv, acc);
          mma_f16_ss(tmem + kColOhi, sw128_desc(v_hi + s * 2048, kSlotBytes / 2, 1024), bdesc,
                     idesc_pv, acc);
        }
        mma_commit(&c.slot_empty[lo % kSlots]);
        mma_commit(&c.slot_empty[hi % kSlots]);
        mma_commit(&c.o_full);
        return true;
      };

      TileInfo cur, prev;
      uint32_t g = 0;
      while (ok && qs.next(cur)) {
        if (cur.seg_first) {
          ok = mbar_wait(&c.q_full, par(nq), abort_flag);
          ++nq;
          if (!ok) break;
        }
        if (g >= 2 && !(ok = mbar_wait(&c.s_empty[g & 1], par((g >> 1) - 1), abort_flag))) break;
        const uint32_t lo = item++, hi = item++;
        if (!(ok = mbar_wait(&c.slot_full[lo % kSlots], par(lo / kSlots), abort_flag))) break;
        if (!(ok = mbar_wait(&c.slot_full[hi % kSlots], par(hi / kSlots), abort_flag))) break;
        tc_fence_after();
        const uint32_t k_lo = ring_base + (lo % kSlots) * kSlotBytes;
        const uint32_t k_hi = ring_base + (hi % kSlots) * kSlotBytes;
        const uint32_t d_s = tmem + kColS + (g & 1) * 64;
#pragma unroll
        for (int s = 0; s < kDim / 16; ++s) {
          const uint32_t a_addr = (s < 8 ? k_lo : k_hi) + ((s >> 2) & 1) * (kSlotBytes / 2) +
                                  (s & 3) * 32;
          const uint32_t b_addr = q_base + (s >> 2) * 8192 + (s & 3) * 32;
          mma_f16_ss(d_s, sw128_desc(a_addr, 16, 1024), sw128_desc(b_addr, 16, 1024), idesc_qk,
                     s > 0 ? 1u : 0u);
        }
        mma_commit(&c.slot_empty[lo % kSlots]);
        mma_commit(&c.slot_empty[hi % kSlots]);
        mma_commit(&c.s_full[g & 1]);
        if (cur.seg_last) mma_commit(&c.q_empty);
        if (g >= 1 && !(ok = issue_pv(prev, g - 1))) break;
        prev = cur;
        ++g;
      }
      if (ok && g >= 1) ok = issue_pv(prev, g - 1);
      if (!ok) {
        // drain: wait (bounded, ignoring the abort flag) for issued MMAs
        mma_commit(&c.drain);
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&c.drain, 0) && global_timer_ns() - t0 < kWaitLimitNs) {
        }
      }
    }
  } else if (warp == 2) {
    // ======================= q producer =====================================
    if (lane == 0) {
      const uint64_t policy = l2_policy_evict_last();
      TileStream qs;
      qs.init(p, c.b_start, c.off_start, c.tiles);
      TileInfo t;
      uint32_t k = 0;
      while (qs.next(t)) {
        if (!t.seg_first) continue;
        if (!mbar_wait(&c.q_empty, par(k) ^ 1u, abort_flag)) break;
        mbar_arrive_expect_tx(&c.q_full, kQBytes);
        for (int r = 0; r < 4; ++r)
          tma_load_3d(sQ + r * 8192, &tm_q, &c.q_full, r * 64, 0, t.b, policy);
        ++k;
      }
    }
  } else if (warp >= 4) {
    // ======================= softmax + epilogue =============================
    const int sub = warp & 3;                 // TMEM sub-partition of this warp
    const int row = sub * 32 + lane;          // token row in S^T / dim row in O^T
    const uint32_t lane_addr = static_cast<uint32_t>(sub * 32) << 16;
    TileStream ts;
    ts.init(p, c.b_start, c.off_start, c.tiles);
    TileInfo t;
    uint32_t g = 0, nseg = 0;
    float m_run0 = -INFINITY, m_run1 = -INFINITY;  // running max, heads 2*lane, 2*lane+1
    float l_part[kHeads];
#pragma unroll
    for (int h = 0; h < kHeads; ++h) l_part[h] = 0.f;
    const float sl2 = p.score_log2;

    while (ts.next(t)) {
      if (t.seg_first) {
        m_run0 = m_run1 = -INFINITY;
#pragma unroll
        for (int h = 0; h < kHeads; ++h) l_part[h] = 0.f;
      }
      // ---- scores of this tile ----------------------------------------
      if (!mbar_wait(&c.s_full[g & 1], par(g >> 1), abort_flag)) break;
      tc_fence_after();
      float s[kHeads];
      {
        uint32_t r[32];
        const uint32_t a = tmem + lane_addr + kColS + (g & 1) * 64;
        tmem_ld32(a, r);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) s[h] = __uint_as_float(r[h]);
        tmem_ld32(a + 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < 32; ++h) s[32 + h] = __uint_as_float(r[h]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.s_empty[g & 1]);

      const int valid = min(kTile, t.L - t.tile * kTile);
      const bool row_ok = row < valid;
#pragma unroll
      for (int h = 0; h < kHeads; ++h) s[h] = row_ok ? s[h] * sl2 : -INFINITY;

      // ---- per-head maximum over the tile's 128 rows --------------------
      {
        float v[kHeads];
#pragma unroll
        for (int h = 0; h < kHeads; ++h) v[h] = s[h];
        reduce_scatter64<true>(v, lane);
        c.red[g & 1][sub][2 * lane] = v[0];
        c.red[g & 1][sub][2 * lane + 1] = v[1];
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.red_full[g & 1]);
      if (!mbar_wait(&c.red_full[g & 1], par(g >> 1), abort_flag)) break;
      float tmax0 = c.red[g & 1][0][2 * lane], tmax1 = c.red[g & 1][0][2 * lane + 1];
#pragma unroll
      for (int w = 1; w < 4; ++w) {
        tmax0 = fmaxf(tmax0, c.red[g & 1][w][2 * lane]);
        tmax1 = fmaxf(tmax1, c.red[g & 1][w][2 * lane + 1]);
      }
      // lazy rescaling: move the reference max only when the tile's max
      // exceeds it by more than the threshold (exact: the factor cancels)
      float m_new0 = m_run0, m_new1 = m_run1, corr0 = 1.f, corr1 = 1.f;
      if (tmax0 > m_run0 + kRescaleThreshold) {
        m_new0 = tmax0;
        corr0 = ex2_approx(m_run0 - tmax0);
      }
      if (tmax1 > m_run1 + kRescaleThreshold) {
        m_new1 = tmax1;
        corr1 = ex2_approx(m_run1 - tmax1);
      }
      m_run0 = m_new0;
      m_run1 = m_new1;
      const bool rescale = __any_sync(0xffffffffu, corr0 != 1.f || corr1 != 1.f);
      c.mv[sub][2 * lane] = m_new0;
      c.mv[sub][2 * lane + 1] = m_new1;
      c.cv[sub][2 * lane] = corr0;
      c.cv[sub][2 * lane + 1] = corr1;
      __syncwarp();

      // ---- probabilities, row sums ---------------------------------------
      uint32_t pk[kHeads / 2];
#pragma unroll
      for (int h = 0; h < kHeads; h += 2) {
        const float2 m2 = *reinterpret_cast<const float2*>(&c.mv[sub][h]);
        const float p0 = ex2_approx(s[h] - m2.x);
        const float p1 = ex2_approx(s[h + 1] - m2.y);
        if (rescale) {
          const float2 c2 = *reinterpret_cast<const float2*>(&c.cv[sub][h]);
          l_part[h] = l_part[h] * c2.x + p0;
          l_part[h + 1] = l_part[h + 1] * c2.y + p1;
        } else {
          l_part[h] += p0;
          l_part[h + 1] += p1;
        }
        pk[h / 2] = pack_bf16x2(p0, p1);
      }

      // ---- P buffer and O are free once the previous tile's PV completed --
      if (g >= 1 && !mbar_wait(&c.o_full, par(g - 1), abort_flag)) break;
      tc_fence_after();
      if (rescale && !t.seg_first) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int cb = 0; cb < 2; ++cb) {
            uint32_t r[32];
            const uint32_t a = tmem + lane_addr + (half ? kColOhi : kColOlo) + cb * 32;
            tmem_ld32(a, r);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              r[j] = __float_as_uint(__uint_as_float(r[j]) * c.cv[sub][cb * 32 + j]);
            tmem_st32(a, r);
          }
        }
        tmem_wait_st();
      }
      {
        const uint32_t rowaddr = smem_u32(sP) + row * 128;
#pragma unroll
        for (int ch = 0; ch < 8; ++ch)
          st_shared_v4(rowaddr + ((ch ^ (row & 7)) << 4), pk[4 * ch], pk[4 * ch + 1],
                       pk[4 * ch + 2], pk[4 * ch + 3]);
      }
      // rows past the sequence end: zero the V rows so 0 * (stale or NaN) never
      // reaches the accumulator
      if (valid < kTile) {
        const uint32_t it = v_item(g, t.cta_last);
        bool ok = mbar_wait(&c.slot_full[it % kSlots], par(it / kSlots), abort_flag);
        ok = ok && mbar_wait(&c.slot_full[(it + 1) % kSlots], par((it + 1) / kSlots), abort_flag);
        if (!ok) break;
        if (!row_ok) {
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint32_t base = smem_u32(sRing) + ((it + hh) % kSlots) * kSlotBytes + row * 128;
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
              for (int ch = 0; ch < 8; ++ch)
                st_shared_v4(base + r * (kSlotBytes / 2) + ch * 16, 0u, 0u, 0u, 0u);
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&c.p_full);

      // ---- epilogue at the end of a segment -------------------------------
      if (t.seg_last) {
        // row sums: reduce the 128 rows' partial sums per head
        {
          float v[kHeads];
#pragma unroll
          for (int h = 0; h < kHeads; ++h) v[h] = l_part[h];
          reduce_scatter64<false>(v, lane);
          c.lred[sub][2 * lane] = v[0];
          c.lred[sub][2 * lane + 1] = v[1];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&c.l_full);
        if (!mbar_wait(&c.l_full, par(nseg), abort_flag)) break;
        const float l0 = c.lred[0][2 * lane] + c.lred[1][2 * lane] + c.lred[2][2 * lane] +
                         c.lred[3][2 * lane];
        const float l1 = c.lred[0][2 * lane + 1] + c.lred[1][2 * lane + 1] +
                         c.lred[2][2 * lane + 1] + c.lred[3][2 * lane + 1];
        // this warp's copy: 1/l in cv, lse (natural log) in mv
        __syncwarp();
        c.cv[sub][2 * lane] = p.out_scale / l0;
        c.cv[sub][2 * lane + 1] = p.out_scale / l1;
        const float lse0 = (m_run0 + lg2_approx(l0)) * kLn2;
        const float lse1 = (m_run1 + lg2_approx(l1)) * kLn2;
        c.mv[sub][2 * lane] = lse0;
        c.mv[sub][2 * lane + 1] = lse1;
        if (sub == 0) {
          if (t.slot >= 0) {
            p.ws_lse[static_cast<int64_t>(t.slot) * kHeads + 2 * lane] = lse0;
            p.ws_lse[static_cast<int64_t>(t.slot) * kHeads + 2 * lane + 1] = lse1;
          } else if (p.lse_out) {
            p.lse_out[t.b * p.lse_sb + 2 * lane] = lse0;
            p.lse_out[t.b * p.lse_sb + 2 * lane + 1] = lse1;
          }
        }
        __syncwarp();
        // O = O^T / l, written row (head-dim index) by row
        if (!mbar_wait(&c.o_full, par(g), abort_flag)) break;
        tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const int d = half * 128 + row;
#pragma unroll
          for (int cb = 0; cb < 2; ++cb) {
            uint32_t r[32];
            tmem_ld32(tmem + lane_addr + (half ? kColOhi : kColOlo) + cb * 32, r);
            tmem_wait_ld();
            if (t.slot >= 0) {
              float* dst = p.ws_o + static_cast<int64_t>(t.slot) * kPartialFloats + d;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int h = cb * 32 + j;
                dst[h * kDim] = __uint_as_float(r[j]) * c.cv[sub][h];
              }
            } else if (p.out_f32) {
              float* dst = static_cast<float*>(p.out) + t.b * p.out_sb + d;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int h = cb * 32 + j;
                dst[h * p.out_sh] = __uint_as_float(r[j]) * c.cv[sub][h];
              }
            } else {
              __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.out) + t.b * p.out_sb + d;
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int h = cb * 32 + j;
                dst[h * p.out_sh] = __float2bfloat16_rn(__uint_as_float(r[j]) * c.cv[sub][h]);
              }
            }
          }
        }
        tc_fence_before();
        ++nseg;
      }
      ++g;
    }
  }

  // ---- teardown ------------------------------------------------------------
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

// ===========================================================================
// Split merge: one CTA per sequence, thread = head-dim index.
// ===========================================================================
// Balanced plan: slot of the i-th CTA (counting from c_first) that holds part of
// a split sequence, or -1 when that CTA's tile range is empty (more CTAs than
// tiles).
__device__ __forceinline__ int balanced_slot(int i, int c_first, int slot_of_first,
                                             long long N, long long G) {
  if (i == 0) return slot_of_first;
  const long long cc = c_first + i;
  const long long lo = (cc * N) / G, hi = ((cc + 1) * N) / G;
  return hi > lo ? static_cast<int>(2 * cc) : -1;
}

__global__ void __launch_bounds__(256) mfa_combine_kernel(const DecodeParams p) {
  const int b = blockIdx.x;
  const int d = threadIdx.x;
  __shared__ float s_lse[64][kHeads + 1];  // per slot (chunked) x head
  __shared__ int s_slot[64];
  __shared__ float s_m[kHeads], s_wsum[kHeads];

  int L = __ldg(p.seq_lens + b);
  if (L < 0 || L > p.cap_tokens) L = 0;  // recorded by the attention kernel
  const int nt = (L + kTile - 1) / kTile;

  // the list of partial slots of this sequence, in plan order
  int nslots = 0;
  int slot_of_first = 0, c_first = 0, c_last = -1;
  long long nt_total = 0;
  if (nt > 0) {
    if (p.num_splits == 0) {
      const long long S = __ldg(p.ws_prefix + b);
      const long long N = __ldg(p.ws_prefix + p.batch);
      const long long G = p.grid;
      nt_total = N;
      auto owner = [&](long long tt) -> int {
        return static_cast<int>(((tt + 1) * G - 1) / N);
      };
      c_first = owner(S);
      c_last = owner(S + nt - 1);
      if (c_first == c_last) return;  // written directly by the attention kernel
      const long long start_first = (static_cast<long long>(c_first) * N) / G;
      slot_of_first = (start_first < S) ? 2 * c_first + 1 : 2 * c_first;
      nslots = c_last - c_first + 1;
    } else {
      const int s = p.num_splits;
      int nonempty = 0;
      for (int j = 0; j < s; ++j) {
        const int lo = static_cast<int>((static_cast<long long>(j) * nt) / s);
        const int hi = static_cast<int>((static_cast<long long>(j + 1) * nt) / s);
        nonempty += hi > lo;
      }
      if (nonempty <= 1) return;
      nslots = s;  // empty units are skipped below
    }
  }

  if (nt == 0) {
    // empty sequence: zeros, lse = -inf
    for (int h = 0; h < kHeads; ++h) {
      if (p.out_f32)
        static_cast<float*>(p.out)[b * p.out_sb + h * p.out_sh + d] = 0.f;
      else
        static_cast<__nv_bfloat16*>(p.out)[b * p.out_sb + h * p.out_sh + d] =
            __float2bfloat16_rn(0.f);
    }
    if (p.lse_out && d < kHeads) p.lse_out[b * p.lse_sb + d] = -INFINITY;
    return;
  }

  // pass over slots in chunks of 64 to find the per-head max and weight sum
  float acc[kHeads];
#pragma unroll
  for (int h = 0; h < kHeads; ++h) acc[h] = 0.f;
  if (d < kHeads) {
    s_m[d] = -INFINITY;
    s_wsum[d] = 0.f;
  }
  __syncthreads();
  // first pass: maxima
  for (int base = 0; base < nslots; base += 64) {
    const int cnt = min(64, nslots - base);
    if (d < cnt) {
      int slot;
      const int i = base + d;
      if (p.num_splits == 0) {
        slot = balanced_slot(i, c_first, slot_of_first, nt_total, p.grid);
      } else {
        const int s = p.num_splits;
        const int lo = static_cast<int>((static_cast<long long>(i) * nt) / s);
        const int hi = static_cast<int>((static_cast<long long>(i + 1) * nt) / s);
        slot = (hi > lo) ? b * s + i : -1;
      }
      s_slot[d] = slot;
    }
    __syncthreads();
    for (int e = d; e < cnt * kHeads; e += blockDim.x) {
      const int i = e / kHeads, h = e % kHeads;
      const int slot = s_slot[i];
      s_lse[i][h] = slot >= 0 ? __ldg(p.ws_lse + static_cast<int64_t>(slot) * kHeads + h)
                              : -INFINITY;
    }
    __syncthreads();
    if (d < kHeads) {
      float m = s_m[d];
      for (int i = 0; i < cnt; ++i) m = fmaxf(m, s_lse[i][d]);
      s_m[d] = m;
    }
    __syncthreads();
  }
  // second pass: weighted sums
  for (int base = 0; base < nslots; base += 64) {
    const int cnt = min(64, nslots - base);
    if (d < cnt) {
      int slot;
      const int i = base + d;
      if (p.num_splits == 0) {
        slot = balanced_slot(i, c_first, slot_of_first, nt_total, p.grid);
      } else {
        const int s = p.num_splits;
        const int lo = static_cast<int>((static_cast<long long>(i) * nt) / s);
        const int hi = static_cast<int>((static_cast<long long>(i + 1) * nt) / s);
        slot = (hi > lo) ? b * s + i : -1;
      }
      s_slot[d] = slot;
    }
    __syncthreads();
    for (int e = d; e < cnt * kHeads; e += blockDim.x) {
      const int i = e / kHeads, h = e % kHeads;
      const int slot = s_slot[i];
      const float l = slot >= 0 ? __ldg(p.ws_lse + static_cast<int64_t>(slot) * kHeads + h)
                                : -INFINITY;
      s_lse[i][h] = (slot >= 0) ? expf(l - s_m[h]) : 0.f;
    }
    __syncthreads();
    if (d < kHeads) {
      float w = s_wsum[d];
      for (int i = 0; i < cnt; ++i) w += s_lse[i][d];
      s_wsum[d] = w;
    }
    for (int i = 0; i < cnt; ++i) {
      const int slot = s_slot[i];
      if (slot < 0) continue;
      const float* src = p.ws_o + static_cast<int64_t>(slot) * kPartialFloats + d;
#pragma unroll
      for (int h = 0; h < kHeads; ++h) acc[h] += s_lse[i][h] * __ldg(src + h * kDim);
    }
    __syncthreads();
  }
#pragma unroll
  for (int h = 0; h < kHeads; ++h) {
    const float o = acc[h] / s_wsum[h];
    if (p.out_f32)
      static_cast<float*>(p.out)[b * p.out_sb + h * p.out_sh + d] = o;
    else
      static_cast<__nv_bfloat16*>(p.out)[b * p.out_sb + h * p.out_sh + d] =
          __float2bfloat16_rn(o);
  }
  if (p.lse_out && d < kHeads) p.lse_out[b * p.lse_sb + d] = s_m[d] + logf(s_wsum[d]);
}

// ===========================================================================
// host-side launch helpers (called from mfa_api.cu)
// ===========================================================================
int decode_smem_bytes() { return kSmemBytes; }

cudaError_t launch_decode(bool paged, const CUtensorMap& tq, const CUtensorMap& tk,
                          const CUtensorMap& tv, const DecodeParams& p, cudaStream_t stream) {
  static thread_local int configured_dev[2] = {-1, -1};
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t err;
  if (configured_dev[paged ? 1 : 0] != dev) {
    err = paged ? cudaFuncSetAttribute(mfa_decode_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes)
                : cudaFuncSetAttribute(mfa_decode_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    if (err != cudaSuccess) return err;
    configured_dev[paged ? 1 : 0] = dev;
  }
  if (paged)
    mfa_decode_kernel<true><<<p.grid, kDecodeThreads, kSmemBytes, stream>>>(tq, tk, tv, p);
  else
    mfa_decode_kernel<false><<<p.grid, kDecodeThreads, kSmemBytes, stream>>>(tq, tk, tv, p);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  mfa_combine_kernel<<<p.batch, 256, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mfa
