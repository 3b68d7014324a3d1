// qproj_kernel.cu -- the MFA low-rank query projection on sm_100a.
//
// Step-3 page, "Key points -> Architecture": queries pass through a 2048-wide
// low-rank bottleneck from the 7168-wide hidden state:  q = (x W_qa) W_qb.
// At decode the batch is small (8 in the long-context workload), so both
// products are weight-streaming GEMMs bound by HBM. They run "swap-AB" on the
// tensor core: the weight matrix is the MMA's A operand (output features on
// M = 128, read MN-major straight from the row-major weight by TMA), the few
// activation rows are the B operand (N = batch padded to 16), the accumulator
// lives in TMEM.
//
//   mode 0 (latent):  C^T = W_qa^T x^T, split over K across CTAs; fp32
//                     partials are merged deterministically by the last CTA of
//                     each output tile, which stores the latent row j as a bf16
//                     high part (row 2j) and a bf16 residual (row 2j+1).
//   mode 1 (up-proj): C^T = W_qb^T L^T with L the 2B interleaved latent rows;
//                     columns 2j and 2j+1 are added in fp32, so the latent enters
//                     with ~16 significant bits at no extra cost (N is padded to
//                     16 columns anyway).

#include "mfa_internal.h"
#include "sm100.cuh"

namespace mfa {

namespace {

constexpr int kGemmThreads = 128;
constexpr int kABytes = 2 * 64 * 128;  // 128 output features x 64 k, bf16 (two 64-wide atoms)

struct __align__(8) GemmCtrl {
  uint64_t full[8], empty[8];
  uint64_t acc_ready;
  uint32_t tmem_base;
  int abort_flag;
  int is_last;
};

__host__ __device__ inline int gemm_stages(int n_cols) {
  const int stage = kABytes + n_cols * 128;
  int s = (200 * 1024) / stage;
  return s > 8 ? 8 : s;
}

__host__ __device__ inline int gemm_tmem_cols(int n_cols) {
  int c = 32;
  while (c < n_cols) c <<= 1;
  return c;
}


// Deterministic split-K merge of latent feature m: for every row j, the sum
// over splits in split order of partials[split][j][m], stored as a bf16 high
// part (row 2j) and a bf16 residual (row 2j + 1). Loads for up to 16 splits
// and kMergeRows rows are all issued before the first add, so the merge costs
// a few L2 round trips rather than one per partial.
constexpr int kMergeSplits = 16;

template <int kMergeRows>
__device__ __forceinline__ void merge_latent(const float* partials, int splits, int B,
                                             int rank, int m, __nv_bfloat16* latent) {
  for (int j0 = 0; j0 < B; j0 += kMergeRows) {
    for (int s0 = 0; s0 < splits; s0 += kMergeSplits) {
      float v[kMergeRows][kMergeSplits];
#pragma unroll
      for (int u = 0; u < kMergeSplits; ++u)
#pragma unroll
        for (int r = 0; r < kMergeRows; ++r)
          v[r][u] = (s0 + u < splits && j0 + r < B)
                        ? __ldcg(partials + (static_cast<int64_t>(s0 + u) * B + j0 + r) * rank + m)
                        : 0.f;
#pragma unroll
      for (int r = 0; r < kMergeRows; ++r) {
        if (j0 + r >= B) break;
        float acc = s0 == 0 ? 0.f : __bfloat162float(latent[static_cast<int64_t>(2 * (j0 + r)) * rank + m]) +
                                        __bfloat162float(latent[static_cast<int64_t>(2 * (j0 + r) + 1) * rank + m]);
#pragma unroll
        for (int u = 0; u < kMergeSplits; ++u) acc += v[r][u];
        const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
        const __nv_bfloat16 lo = __float2bfloat16_rn(acc - __bfloat162float(hi));
        latent[static_cast<int64_t>(2 * (j0 + r)) * rank + m] = hi;
        latent[static_cast<int64_t>(2 * (j0 + r) + 1) * rank + m] = lo;
      }
    }
  }
}

// The fused kernel's merge: 128 threads, thread = 4 adjacent features (16-byte
// loads) x 2 latent rows; all splits of both rows are loaded before the first
// add, 8 splits at a time, and summed in split order in fp32. Needs B <= 8,
// rank a multiple of 4 and 16-byte aligned partials.
constexpr int kMergeBatch = 8;
__device__ __forceinline__ void merge_latent_x4(const float* partials, int splits, int B, int rank,
                                                int m_tile0, int etid, __nv_bfloat16* latent) {
  const int m = m_tile0 + (etid & 31) * 4;
  const int r0 = (etid >> 5) * 2;
  float4 acc[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
  for (int s0 = 0; s0 < splits; s0 += kMergeBatch) {
    float4 v[2][kMergeBatch];
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr)
        v[rr][u] = (s0 + u < splits && r0 + rr < B)
                       ? __ldcg(reinterpret_cast<const float4*>(
                             partials + (static_cast<int64_t>(s0 + u) * B + r0 + rr) * rank + m))
                       : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kMergeBatch; ++u)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        if (s0 + u >= splits) continue;
        acc[rr].x += v[rr][u].x;
        acc[rr].y += v[rr][u].y;
        acc[rr].z += v[rr][u].z;
        acc[rr].w += v[rr][u].w;
      }
  }
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    const int r = r0 + rr;
    if (r >= B) break;
    const float a[4] = {acc[rr].x, acc[rr].y, acc[rr].z, acc[rr].w};
    __nv_bfloat16 hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      hi[e] = __float2bfloat16_rn(a[e]);
      lo[e] = __float2bfloat16_rn(a[e] - __bfloat162float(hi[e]));
    }
    uint2 h, l;
    h.x = static_cast<uint32_t>(__bfloat16_as_ushort(hi[0])) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi[1])) << 16);
    h.y = static_cast<uint32_t>(__bfloat16_as_ushort(hi[2])) | (static_cast<uint32_t>(__bfloat16_as_ushort(hi[3])) << 16);
    l.x = static_cast<uint32_t>(__bfloat16_as_ushort(lo[0])) | (static_cast<uint32_t>(__bfloat16_as_ushort(lo[1])) << 16);
    l.y = static_cast<uint32_t>(__bfloat16_as_ushort(lo[2])) | (static_cast<uint32_t>(__bfloat16_as_ushort(lo[3])) << 16);
    *reinterpret_cast<uint2*>(latent + static_cast<int64_t>(2 * r) * rank + m) = h;
    *reinterpret_cast<uint2*>(latent + static_cast<int64_t>(2 * r + 1) * rank + m) = l;
  }
}
}  // namespace

__global__ void __launch_bounds__(kGemmThreads, 1)
    mfa_qproj_kernel(const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_act,
                     const __grid_constant__ CUtensorMap tm_w2, const QprojParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int n_cols = p.n_cols;
  const int stages = gemm_stages(n_cols);
  const int stage_bytes = kABytes + n_cols * 128;
  GemmCtrl& c = *reinterpret_cast<GemmCtrl*>(smem + stages * stage_bytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m_tile = blockIdx.x;
  const int split = blockIdx.y;
  const int kb0 = static_cast<int>((static_cast<long long>(split) * p.k_blocks) / p.splits);
  const int kb1 = static_cast<int>((static_cast<long long>(split + 1) * p.k_blocks) / p.splits);
  const int nkb = kb1 - kb0;
  const uint32_t tcols = gemm_tmem_cols(n_cols);

  if (tid == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&c.full[i], 1);
      mbar_init(&c.empty[i], 1);
    }
    mbar_init(&c.acc_ready, 1);
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched with programmatic dependent launch: the set-up above may overlap
  // the previous kernel's tail; nothing in global memory is touched before it
  // has completed
  griddep_wait();
  // A kernel launched after this one with programmatic dependent launch (the
  // decode attention after the up-projection, the key/value merge after the
  // append projection) may set up as this grid's CTAs finish; it reads this
  // grid's results only after it has completed. The trigger follows the
  // dependency wait, so that kernel starts only once every kernel before this
  // one has completed (the projection -> attention call relies on it).
  griddep_launch_dependents();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort_flag = &c.abort_flag;

  if (warp == 0 && lane == 0) {
    // ---------------- producer ----------------
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_a = l2_policy_evict_last();
    // mode 2: tiles from m_half on are the second weight's (W_v)
    const bool second = p.mode == 2 && m_tile >= p.m_half;
    const CUtensorMap* wm = second ? &tm_w2 : &tm_w;
    const int wcol = (second ? m_tile - p.m_half : m_tile) * 128;
    tma_prefetch_desc(wm);
    tma_prefetch_desc(&tm_act);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % stages;
      if (!mbar_wait(&c.empty[s], ((i / stages) & 1) ^ 1, abort_flag)) break;
      uint8_t* st = smem + s * stage_bytes;
      mbar_arrive_expect_tx(&c.full[s], stage_bytes);
      const int kb = kb0 + i;
      tma_load_2d(st, wm, &c.full[s], wcol, kb * 64, pol_w);
      tma_load_2d(st + kABytes / 2, wm, &c.full[s], wcol + 64, kb * 64, pol_w);
      tma_load_2d(st + kABytes, &tm_act, &c.full[s], kb * 64, 0, pol_a);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp, one elected lane issues ----------------
    const uint32_t idesc = idesc_f16(128, n_cols, 1, 1, 0);
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nkb; ++i) {
      if (!mbar_wait_warp(&c.full[s], ph, abort_flag)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + s * stage_bytes);
      const uint32_t b = a + kABytes;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_f16_ss_warp(tmem, sw128_desc(a + k * 2048, kABytes / 2, 1024),
                        sw128_desc(b + k * 32, 16, 1024), idesc, (i > 0 || k > 0) ? 1u : 0u);
      mma_commit_warp(&c.empty[s]);
      if (++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    }
    mma_commit_warp(&c.acc_ready);
  }

  // ---------------- epilogue: thread = output feature row ----------------
  __syncwarp();
  const bool ready = mbar_wait(&c.acc_ready, 0, abort_flag) && nkb > 0;
  tc_fence_after();
  const int m = m_tile * 128 + warp * 32 + lane;
  const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const int B = p.batch;
  if (ready) {
    if (p.mode == 0 || p.mode == 2) {
      for (int cb = 0; cb < n_cols; cb += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + cb, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (cb + j < B)
            p.partials[(static_cast<int64_t>(split) * B + cb + j) * p.m_total + m] =
                __uint_as_float(r[j]);
      }
    } else {
      // latent rows are interleaved (2j = high part, 2j+1 = residual), so
      // q[j] = C[:, 2j] + C[:, 2j+1]: both columns sit in the same 16-column load
      for (int cb = 0; cb < n_cols; cb += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + cb, r);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int row = cb / 2 + jj;
          if (row < B)
            p.q_out[static_cast<int64_t>(row) * p.q_stride + m] =
                __float2bfloat16_rn(__uint_as_float(r[2 * jj]) + __uint_as_float(r[2 * jj + 1]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, tcols);

  if (p.mode == 0 && ready) {
    // deterministic split-K merge by the last CTA to finish this output tile
    // (one acquire-release add per CTA, as in the fused kernel)
    __syncthreads();
    if (tid == 0) {
      const int prev = atom_add_acq_rel_gpu(p.counters + m_tile, 1);
      c.is_last = (prev == p.splits - 1);
    }
    __syncthreads();
    if (c.is_last) {
      merge_latent<2>(p.partials, p.splits, B, p.m_total, m, p.latent);
      if (tid == 0) p.counters[m_tile] = 0;
    }
  }
}

// ===========================================================================
// Both GEMMs in one persistent kernel, for small batches. CTA i < m1_tiles x
// splits computes a split-K part of the latent GEMM as above; CTA i <
// m2_tiles owns output tile i of the up-projection. An up-projection stage
// holds a weight tile and the matching 64-wide slice of the latent, loaded
// separately: the weight parts are issued as soon as slots free, so the ring
// fills with the second GEMM's weights while the latent is still being
// formed, and the latent parts follow once every latent tile is complete (a
// bounded wait on the latent-ready count, taken only when the ring is full).
// Grid = at most one CTA per SM, so every CTA is resident while others wait.
// The weights come through 3-D maps (64 features, k, 64-feature chunk): one
// TMA op per 128 x 64 tile. Warp 0 loads, warp 1 issues the products; warps
// 2-5 (TMEM lane quarters warp & 3) run the epilogues and synchronise only
// among themselves.
// ===========================================================================
namespace {

constexpr int kFusedThreads = 192;
constexpr int kEpiThreads = 128;
constexpr int kFusedTmemCols = 64;  // latent accumulator at 0, output accumulator at 32

__device__ __forceinline__ void epi_sync() {  // warps 2-5 only
  asm volatile("bar.sync 1, %0;" ::"n"(kEpiThreads) : "memory");
}

struct __align__(8) FusedCtrl {
  uint64_t full[16], empty[16];
  uint64_t acc1, acc2;
  uint32_t tmem_base;
  int abort_flag;
  int is_last;
};

__host__ __device__ inline int fused_stage_bytes(int n1, int n2) {
  return kABytes + (n1 > n2 ? n1 : n2) * 128;
}

__host__ __device__ inline int fused_stages(int stage_bytes) {
  const int s = (218 * 1024) / stage_bytes;
  return s > 16 ? 16 : s;
}

}  // namespace

__global__ void __launch_bounds__(kFusedThreads, 1)
    mfa_qproj_fused_kernel(const __grid_constant__ CUtensorMap tm_wa,
                           const __grid_constant__ CUtensorMap tm_x,
                           const __grid_constant__ CUtensorMap tm_wb,
                           const __grid_constant__ CUtensorMap tm_lat, const QprojFusedParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int stage_bytes = fused_stage_bytes(p.n1, p.n2);
  const int stages = fused_stages(stage_bytes);
  FusedCtrl& c = *reinterpret_cast<FusedCtrl*>(smem + stages * stage_bytes);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool has1 = static_cast<int>(blockIdx.x) < p.m1_tiles * p.splits;
  const int tile1 = blockIdx.x % p.m1_tiles;
  const int split = blockIdx.x / p.m1_tiles;
  const int kb0 = static_cast<int>((static_cast<long long>(split) * p.k1_blocks) / p.splits);
  const int kb1 = static_cast<int>((static_cast<long long>(split + 1) * p.k1_blocks) / p.splits);
  const bool has2 = static_cast<int>(blockIdx.x) < p.m2_tiles;
  const int tile2 = blockIdx.x;

  if (tid == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&c.full[i], 1);
      mbar_init(&c.empty[i], 1);
    }
    mbar_init(&c.acc1, 1);
    mbar_init(&c.acc2, 1);
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, kFusedTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // launched with programmatic dependent launch: the set-up above may overlap
  // the previous kernel's tail; nothing in global memory is touched before it
  // has completed
  griddep_wait();
  // A kernel launched after this one with programmatic dependent launch (the
  // decode attention of mfa_qproj_decode_attention) may start as this grid's
  // CTAs finish. The trigger follows the dependency wait: once it fires in
  // every CTA, every kernel before this one has completed, so that attention
  // kernel reads the lengths, the caches and its workspace at once and waits
  // for this grid only before it reads q.
  griddep_launch_dependents();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort_flag = &c.abort_flag;

  if (warp == 0) {
    // ---------------- producer: the whole warp, one elected lane issues ----------------
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_a = l2_policy_evict_last();
    if (lane == 0) {
      tma_prefetch_desc(&tm_wa);
      tma_prefetch_desc(&tm_x);
      tma_prefetch_desc(&tm_wb);
      tma_prefetch_desc(&tm_lat);
    }
    __syncwarp();
    int s = 0;  // ring slot and phase of the next stage
    uint32_t ph = 0;
    bool ok = true;
    if (has1) {
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!(ok = mbar_wait_warp(&c.empty[s], ph ^ 1u, abort_flag))) break;
        uint8_t* st = smem + s * stage_bytes;
        mbar_arrive_expect_tx_warp(&c.full[s], kABytes + p.n1 * 128);
        tma_load_3d_warp(st, &tm_wa, &c.full[s], 0, kb * 64, 2 * tile1, pol_w);
        tma_load_2d_warp(st + kABytes, &tm_x, &c.full[s], kb * 64, 0, pol_a);
        if (++s == stages) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
    if (has2 && ok) {
      int ls = s;          // slot of the next latent part
      int lat_issued = 0;  // k-blocks whose latent part is issued
      bool lat_ready = false;
      // latent parts of k-blocks [lat_issued, kb_end)
      auto issue_latent = [&](int kb_end) {
        for (; lat_issued < kb_end; ++lat_issued) {
          tma_load_2d_warp(smem + ls * stage_bytes + kABytes, &tm_lat, &c.full[ls],
                           lat_issued * 64, 0, pol_a);
          if (++ls == stages) ls = 0;
        }
      };
      // the whole latent exists once every latent tile is merged (bounded);
      // every lane reads the same words, so the warp leaves the loop together
      auto await_latent = [&]() -> bool {
        const int* done = p.counters + kQprojDone;
        const uint64_t t0 = global_timer_ns();
        bool good = true;
        while (ld_acquire_gpu(done) < p.m1_tiles) {  // acquires the latent tiles
          if (*abort_flag) {
            good = false;
            break;
          }
          if (global_timer_ns() - t0 > kWaitLimitNs) {
            if (lane == 0) {
              record_error(6 /* MFA_ERR_TIMEOUT */);
              *abort_flag = 1;
            }
            good = false;
            break;
          }
        }
        if (!__all_sync(0xffffffffu, good)) return false;
        fence_proxy_async_global();  // the acquired latent, for the TMA reads that follow
        // count this CTA as having seen the latent; the last one (after all
        // latent tiles and every other reader) returns the count to zero
        if (lane == 0 && atomicAdd(p.counters + kQprojDone, 1) == p.m1_tiles + p.m2_tiles - 1)
          p.counters[kQprojDone] = 0;
        __syncwarp();
        return true;
      };
      for (int kb = 0; kb < p.k2_blocks && ok; ++kb) {
        if (!lat_ready && kb >= stages) {
          // the ring is full of weight parts: the products need the latent now
          if (!(ok = await_latent())) break;
          lat_ready = true;
          issue_latent(kb);
        }
        if (!(ok = mbar_wait_warp(&c.empty[s], ph ^ 1u, abort_flag))) break;
        uint8_t* st = smem + s * stage_bytes;
        mbar_arrive_expect_tx_warp(&c.full[s], kABytes + p.n2 * 128);
        tma_load_3d_warp(st, &tm_wb, &c.full[s], 0, kb * 64, 2 * tile2, pol_w);
        if (lat_ready) issue_latent(kb + 1);
        if (++s == stages) {
          s = 0;
          ph ^= 1u;
        }
      }
      if (ok && !lat_ready && await_latent()) issue_latent(p.k2_blocks);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp, one elected lane issues ----------------
    const uint32_t idesc1 = idesc_f16(128, p.n1, 1, 1, 0);
    const uint32_t idesc2 = idesc_f16(128, p.n2, 1, 1, 0);
    int s = 0;
    uint32_t ph = 0;
    auto next = [&]() {
      if (++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    };
    bool ok = true;
    if (has1) {
      for (int kb = kb0; kb < kb1; ++kb, next()) {
        if (!(ok = mbar_wait_warp(&c.full[s], ph, abort_flag))) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * stage_bytes);
        const uint32_t b = a + kABytes;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_f16_ss_warp(tmem, sw128_desc(a + k * 2048, kABytes / 2, 1024),
                          sw128_desc(b + k * 32, 16, 1024), idesc1, (kb > kb0 || k > 0) ? 1u : 0u);
        mma_commit_warp(&c.empty[s]);
      }
      mma_commit_warp(&c.acc1);
    }
    if (has2 && ok) {
      for (int kb = 0; kb < p.k2_blocks; ++kb, next()) {
        if (!mbar_wait_warp(&c.full[s], ph, abort_flag)) break;
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * stage_bytes);
        const uint32_t b = a + kABytes;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          mma_f16_ss_warp(tmem + 32, sw128_desc(a + k * 2048, kABytes / 2, 1024),
                          sw128_desc(b + k * 32, 16, 1024), idesc2, (kb > 0 || k > 0) ? 1u : 0u);
        mma_commit_warp(&c.empty[s]);
      }
    }
    if (has2) mma_commit_warp(&c.acc2);
  }
  __syncwarp();

  // ---------------- epilogues: thread = output feature row ----------------
  const int quarter = warp & 3;  // TMEM lanes 32 quarter .. 32 quarter + 31
  const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
  const int etid = tid - 64;     // 0 .. 127 in warps 2-5
  const int B = p.batch;
  if (warp >= 2 && has1) {
    const bool ready = mbar_wait(&c.acc1, 0, abort_flag);
    tc_fence_after();
    const int m = tile1 * 128 + quarter * 32 + lane;
    if (ready) {
      for (int cb = 0; cb < p.n1; cb += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + cb, r);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (cb + j < B)
            p.partials[(static_cast<int64_t>(split) * B + cb + j) * p.rank + m] =
                __uint_as_float(r[j]);
      }
    }
    // deterministic split-K merge by the last CTA of this latent tile: one
    // acquire-release add per CTA (its release half publishes this CTA's
    // partial, made CTA-wide by the barrier; its acquire half the others')
    epi_sync();
    if (etid == 0) {
      const int prev = atom_add_acq_rel_gpu(p.counters + tile1, 1);
      c.is_last = (prev == p.splits - 1);
    }
    epi_sync();
    if (c.is_last) {
      merge_latent_x4(p.partials, p.splits, B, p.rank, tile1 * 128, etid, p.latent);
      epi_sync();
      if (etid == 0) {
        p.counters[tile1] = 0;
        red_add_release_gpu(p.counters + kQprojDone, 1);  // this latent tile is complete
      }
    }
  }
  if (warp >= 2 && has2) {
    const bool ready = mbar_wait(&c.acc2, 0, abort_flag);
    tc_fence_after();
    const int m = tile2 * 128 + quarter * 32 + lane;
    if (ready && !*abort_flag) {
      // latent rows are interleaved (2j = high part, 2j+1 = residual)
      for (int cb = 0; cb < p.n2; cb += 16) {
        uint32_t r[16];
        tmem_ld16(taddr + 32 + cb, r);
        tmem_wait_ld();
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int row = cb / 2 + jj;
          if (row < B)
            p.q_out[static_cast<int64_t>(row) * p.q_stride + m] =
                __float2bfloat16_rn(__uint_as_float(r[2 * jj]) + __uint_as_float(r[2 * jj + 1]));
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, kFusedTmemCols);
}

// Launch with programmatic dependent launch (the kernel waits for the
// previous kernel on the stream before it touches global memory).
template <typename Kernel, typename... Args>
static cudaError_t launch_pdl_qp(Kernel kernel, dim3 grid, dim3 block, size_t smem,
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

int qproj_fused_smem_bytes(int n1, int n2) {
  const int stage_bytes = fused_stage_bytes(n1, n2);
  return fused_stages(stage_bytes) * stage_bytes + static_cast<int>(sizeof(FusedCtrl)) + 1024;
}

bool qproj_fused_fits(int n1, int n2, int k2_blocks) {
  (void)k2_blocks;
  return n1 <= 32 && n2 <= 32 && fused_stages(fused_stage_bytes(n1, n2)) >= 4;
}

cudaError_t launch_qproj_fused(const CUtensorMap& twa, const CUtensorMap& tx,
                               const CUtensorMap& twb, const CUtensorMap& tl,
                               const QprojFusedParams& p, int grid, cudaStream_t stream) {
  const int smem = qproj_fused_smem_bytes(p.n1, p.n2);
  cudaError_t err = cudaFuncSetAttribute(mfa_qproj_fused_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  return launch_pdl_qp(mfa_qproj_fused_kernel, dim3(grid), dim3(kFusedThreads),
                       static_cast<size_t>(smem), stream, twa, tx, twb, tl, p);
}

int qproj_smem_bytes(int n_cols) {
  return gemm_stages(n_cols) * (kABytes + n_cols * 128) + static_cast<int>(sizeof(GemmCtrl)) +
         1024;
}

cudaError_t launch_qproj(const CUtensorMap& tw, const CUtensorMap& ta, const QprojParams& p,
                         int m_tiles, cudaStream_t stream) {
  const int smem = qproj_smem_bytes(p.n_cols);
  cudaError_t err =
      cudaFuncSetAttribute(mfa_qproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  dim3 grid(m_tiles, p.mode == 1 ? 1 : p.splits);
  const cudaError_t e = launch_pdl_qp(mfa_qproj_kernel, grid, dim3(kGemmThreads),
                                      static_cast<size_t>(smem), stream, tw, ta, tw, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// ===========================================================================
// Key/value append: the projection x [W_k | W_v] as split-K partials (the GEMM
// above in mode 2, tiles of W_k then W_v), then a merge kernel in which a
// thread owns one (sequence, feature) output: it sums the splits in order (as
// deterministic as the latent merge) and stores the value into the cache row
// of the sequence's new token -- the nearest bf16, or the E4M3 code nearest to
// value / scale (saturating) for an FP8 cache -- through the page table when
// there is one. Positions and page ids are checked; a bad one is recorded as
// MFA_ERR_BAD_INDEX and its row is not written.
// ===========================================================================
constexpr int kMergeThreads = 256;
constexpr int kAppendSplitBatch = 8;  // partial loads in flight per thread

__global__ void __launch_bounds__(kMergeThreads)
    mfa_kv_merge_kernel(const KvAppendParams p) {
  griddep_wait();  // the partials of the projection kernel
  constexpr int kFeat = 2 * kDim;
  const int64_t o = static_cast<int64_t>(blockIdx.x) * kMergeThreads + threadIdx.x;
  if (o >= static_cast<int64_t>(p.batch) * kFeat) return;
  const int b = static_cast<int>(o / kFeat);
  const int f = static_cast<int>(o % kFeat);
  float acc = 0.f;
  for (int s0 = 0; s0 < p.splits; s0 += kAppendSplitBatch) {
    float v[kAppendSplitBatch];
#pragma unroll
    for (int u = 0; u < kAppendSplitBatch; ++u)
      v[u] = s0 + u < p.splits
                 ? __ldcg(p.partials + (static_cast<int64_t>(s0 + u) * p.batch + b) * kFeat + f)
                 : 0.f;
#pragma unroll
    for (int u = 0; u < kAppendSplitBatch; ++u)
      if (s0 + u < p.splits) acc += v[u];
  }
  const bool is_v = f >= kDim;
  const int d = is_v ? f - kDim : f;
  const int t = p.positions[b];
  int64_t row;  // element offset of the new token's row
  if (p.page_table) {
    if (t < 0 || t >= p.max_pages * p.page_size) {
      record_error(5 /* MFA_ERR_BAD_INDEX */);
      return;
    }
    const int page = p.page_table[static_cast<int64_t>(b) * p.pt_stride + t / p.page_size];
    if (page < 0 || page >= p.num_pages) {
      record_error(5 /* MFA_ERR_BAD_INDEX */);
      return;
    }
    row = static_cast<int64_t>(page) * p.cache_bs + static_cast<int64_t>(t % p.page_size) * p.cache_ts;
  } else {
    if (t < 0 || t >= p.cap_tokens) {
      record_error(5 /* MFA_ERR_BAD_INDEX */);
      return;
    }
    row = static_cast<int64_t>(b) * p.cache_bs + static_cast<int64_t>(t) * p.cache_ts;
  }
  void* cache = is_v ? p.v_cache : p.k_cache;
  if (p.fp8) {
    const float scaled = acc / (is_v ? p.v_scale : p.k_scale);
    static_cast<uint8_t*>(cache)[row + d] =
        static_cast<uint8_t>(__nv_cvt_float_to_fp8(scaled, __NV_SATFINITE, __NV_E4M3));
  } else {
    static_cast<__nv_bfloat16*>(cache)[row + d] = __float2bfloat16_rn(acc);
  }
}

// ===========================================================================
// Output projection y = o W_o (stream-K GEMM + in-order merge, below).
// ===========================================================================
// ---------------------------------------------------------------------------
// Stream-K output projection: the (tile, k-block) units, tile-major, are cut
// into gridDim.x equal contiguous runs, one per CTA, so every SM streams the
// same share of W_o (an even split per tile would leave SMs idle: 56 tiles).
// A run crosses at most one tile boundary (tiles <= CTAs), so a CTA has one or
// two segments, accumulated in two TMEM buffers; each segment's fp32 partial
// goes to slot 2 * cta + segment. The merge sums, per output, the slots of the
// CTAs whose runs cover its tile, in CTA order.
// ---------------------------------------------------------------------------
struct StreamKRun {
  long long u0, u1;  // units [u0, u1) of this CTA
};

__host__ __device__ inline StreamKRun streamk_run(int cta, long long units, int ctas) {
  return {static_cast<long long>(cta) * units / ctas,
          static_cast<long long>(cta + 1) * units / ctas};
}

__global__ void __launch_bounds__(kGemmThreads, 1)
    mfa_streamk_gemm_kernel(const __grid_constant__ CUtensorMap tm_w,
                            const __grid_constant__ CUtensorMap tm_act, const QprojParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int n_cols = p.n_cols;
  const int stages = gemm_stages(n_cols);
  const int stage_bytes = kABytes + n_cols * 128;
  GemmCtrl& c = *reinterpret_cast<GemmCtrl*>(smem + stages * stage_bytes);
  __shared__ uint64_t seg_ready[2];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int KB = p.k_blocks;
  const long long units = static_cast<long long>(p.m_total / 128) * KB;
  const StreamKRun run = streamk_run(blockIdx.x, units, gridDim.x);
  const int nunits = static_cast<int>(run.u1 - run.u0);
  // segment boundary: the first unit of the run's second tile (if any)
  const long long split_u = (run.u0 / KB + 1) * KB;
  const int nseg = nunits <= 0 ? 0 : (run.u1 > split_u ? 2 : 1);
  const uint32_t tcols = gemm_tmem_cols(n_cols);

  if (tid == 0) {
    for (int i = 0; i < stages; ++i) {
      mbar_init(&c.full[i], 1);
      mbar_init(&c.empty[i], 1);
    }
    mbar_init(&seg_ready[0], 1);
    mbar_init(&seg_ready[1], 1);
    c.abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&c.tmem_base, 2 * tcols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = c.tmem_base;
  volatile int* abort_flag = &c.abort_flag;

  if (warp == 0) {
    // ---------------- producer: the whole warp, one elected lane issues ----------------
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_a = l2_policy_evict_last();
    if (lane == 0) {
      tma_prefetch_desc(&tm_w);
      tma_prefetch_desc(&tm_act);
    }
    __syncwarp();
    int s = 0;
    uint32_t ph = 0;
    for (long long u = run.u0; u < run.u1; ++u) {
      if (!mbar_wait_warp(&c.empty[s], ph ^ 1u, abort_flag)) break;
      uint8_t* st = smem + s * stage_bytes;
      const int tile = static_cast<int>(u / KB), kb = static_cast<int>(u % KB);
      mbar_arrive_expect_tx_warp(&c.full[s], stage_bytes);
      tma_load_2d_warp(st, &tm_w, &c.full[s], tile * 128, kb * 64, pol_w);
      tma_load_2d_warp(st + kABytes / 2, &tm_w, &c.full[s], tile * 128 + 64, kb * 64, pol_w);
      tma_load_2d_warp(st + kABytes, &tm_act, &c.full[s], kb * 64, 0, pol_a);
      if (++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: the whole warp, one elected lane issues ----------------
    const uint32_t idesc = idesc_f16(128, n_cols, 1, 1, 0);
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (long long u = run.u0; u < run.u1 && ok; ++u) {
      const int seg = u >= split_u ? 1 : 0;
      const bool first = u == run.u0 || u == split_u;
      if (!(ok = mbar_wait_warp(&c.full[s], ph, abort_flag))) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + s * stage_bytes);
      const uint32_t b = a + kABytes;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_f16_ss_warp(tmem + seg * tcols, sw128_desc(a + k * 2048, kABytes / 2, 1024),
                        sw128_desc(b + k * 32, 16, 1024), idesc, (!first || k > 0) ? 1u : 0u);
      mma_commit_warp(&c.empty[s]);
      if (u + 1 == run.u1 || u + 1 == split_u) mma_commit_warp(&seg_ready[seg]);
      if (++s == stages) {
        s = 0;
        ph ^= 1u;
      }
    }
  }
  __syncwarp();

  // ---------------- epilogue: thread = output feature row of the tile ----------------
  const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const int ml = warp * 32 + lane;
  const int B = p.batch;
  for (int seg = 0; seg < nseg; ++seg) {
    const bool ready = mbar_wait(&seg_ready[seg], 0, abort_flag);
    tc_fence_after();
    if (!ready) break;
    float* dst = p.partials + (static_cast<int64_t>(2 * blockIdx.x + seg) * B) * 128 + ml;
    for (int cb = 0; cb < n_cols; cb += 16) {
      uint32_t r[16];
      tmem_ld16(taddr + seg * tcols + cb, r);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (cb + j < B) dst[static_cast<int64_t>(cb + j) * 128] = __uint_as_float(r[j]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) tmem_dealloc(tmem, 2 * tcols);
}

// The CTA whose run holds unit u (runs as in streamk_run).
__device__ __forceinline__ int streamk_owner(long long u, long long units, int ctas) {
  int c = static_cast<int>((u * ctas) / units);
  while (c + 1 < ctas && streamk_run(c + 1, units, ctas).u0 <= u) ++c;
  while (c > 0 && streamk_run(c, units, ctas).u0 > u) --c;
  return c;
}

__global__ void __launch_bounds__(kMergeThreads)
    mfa_streamk_merge_kernel(const float* partials, int ctas, int k_blocks, int batch, int n,
                             __nv_bfloat16* y, int64_t y_stride) {
  griddep_wait();  // the partials of the stream-K kernel
  const int64_t o = static_cast<int64_t>(blockIdx.x) * kMergeThreads + threadIdx.x;
  if (o >= static_cast<int64_t>(batch) * n) return;
  const int b = static_cast<int>(o / n);
  const int f = static_cast<int>(o % n);
  const int tile = f / 128, ml = f % 128;
  const long long units = static_cast<long long>(n / 128) * k_blocks;
  const long long t0 = static_cast<long long>(tile) * k_blocks;
  const int c_lo = streamk_owner(t0, units, ctas);
  const int c_hi = streamk_owner(t0 + k_blocks - 1, units, ctas);
  float acc = 0.f;
  for (int cta = c_lo; cta <= c_hi; ++cta) {
    // the segment of this CTA's run that lies in the tile: its second one if
    // the run began in an earlier tile
    const int seg = streamk_run(cta, units, ctas).u0 < t0 ? 1 : 0;
    acc += __ldcg(partials + (static_cast<int64_t>(2 * cta + seg) * batch + b) * 128 + ml);
  }
  y[static_cast<int64_t>(b) * y_stride + f] = __float2bfloat16_rn(acc);
}

cudaError_t launch_out_proj(const CUtensorMap& tw, const CUtensorMap& ta, const QprojParams& pg,
                            __nv_bfloat16* y, int64_t y_stride, cudaStream_t stream) {
  const int smem = qproj_smem_bytes(pg.n_cols);
  cudaError_t err =
      cudaFuncSetAttribute(mfa_qproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  err = cudaFuncSetAttribute(mfa_streamk_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             smem);
  if (err != cudaSuccess) return err;
  // pg.splits carries the stream-K grid (CTAs, at least the number of tiles)
  mfa_streamk_gemm_kernel<<<pg.splits, kGemmThreads, smem, stream>>>(tw, ta, pg);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t outputs = static_cast<int64_t>(pg.batch) * pg.m_total;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((outputs + kMergeThreads - 1) / kMergeThreads));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mfa_streamk_merge_kernel, static_cast<const float*>(pg.partials),
                            pg.splits, pg.k_blocks, pg.batch, pg.m_total, y, y_stride);
}

cudaError_t launch_kv_append(const CUtensorMap& twk, const CUtensorMap& twv, const CUtensorMap& tx,
                             const QprojParams& pg, const KvAppendParams& pm, cudaStream_t stream) {
  const int smem = qproj_smem_bytes(pg.n_cols);
  cudaError_t err =
      cudaFuncSetAttribute(mfa_qproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (err != cudaSuccess) return err;
  mfa_qproj_kernel<<<dim3(2 * pg.m_half, pg.splits), kGemmThreads, smem, stream>>>(twk, tx, twv, pg);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const int64_t outputs = static_cast<int64_t>(pm.batch) * 2 * kDim;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((outputs + kMergeThreads - 1) / kMergeThreads));
  cfg.blockDim = dim3(kMergeThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, mfa_kv_merge_kernel, pm);
}

}  // namespace mfa
