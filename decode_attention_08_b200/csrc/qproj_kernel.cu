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

}  // namespace

__global__ void __launch_bounds__(kGemmThreads, 1)
    mfa_qproj_kernel(const __grid_constant__ CUtensorMap tm_w,
                     const __grid_constant__ CUtensorMap tm_act, const QprojParams p) {
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
  const uint32_t tmem = c.tmem_base;
  volatile int* abort_flag = &c.abort_flag;

  if (warp == 0 && lane == 0) {
    // ---------------- producer ----------------
    const uint64_t pol_w = l2_policy_evict_first();
    const uint64_t pol_a = l2_policy_evict_last();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_act);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % stages;
      if (!mbar_wait(&c.empty[s], ((i / stages) & 1) ^ 1, abort_flag)) break;
      uint8_t* st = smem + s * stage_bytes;
      mbar_arrive_expect_tx(&c.full[s], stage_bytes);
      const int kb = kb0 + i;
      tma_load_2d(st, &tm_w, &c.full[s], m_tile * 128, kb * 64, pol_w);
      tma_load_2d(st + kABytes / 2, &tm_w, &c.full[s], m_tile * 128 + 64, kb * 64, pol_w);
      tma_load_2d(st + kABytes, &tm_act, &c.full[s], kb * 64, 0, pol_a);
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_f16(128, n_cols, 1, 1, 0);
    for (int i = 0; i < nkb; ++i) {
      const int s = i % stages;
      if (!mbar_wait(&c.full[s], (i / stages) & 1, abort_flag)) break;
      tc_fence_after();
      const uint32_t a = smem_u32(smem + s * stage_bytes);
      const uint32_t b = a + kABytes;
#pragma unroll
      for (int k = 0; k < 4; ++k)
        mma_f16_ss(tmem, sw128_desc(a + k * 2048, kABytes / 2, 1024), sw128_desc(b + k * 32, 16, 1024),
                   idesc, (i > 0 || k > 0) ? 1u : 0u);
      mma_commit(&c.empty[s]);
    }
    mma_commit(&c.acc_ready);
  }

  // ---------------- epilogue: thread = output feature row ----------------
  __syncwarp();
  const bool ready = mbar_wait(&c.acc_ready, 0, abort_flag) && nkb > 0;
  tc_fence_after();
  const int m = m_tile * 128 + warp * 32 + lane;
  const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  const int B = p.batch;
  if (ready) {
    if (p.mode == 0) {
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
    __threadfence();
    __syncthreads();
    if (tid == 0) {
      const int prev = atomicAdd(p.counters + m_tile, 1);
      c.is_last = (prev == p.splits - 1);
    }
    __syncthreads();
    if (c.is_last) {
      __threadfence();
      for (int j = 0; j < B; ++j) {
        float acc = 0.f;
        for (int s = 0; s < p.splits; ++s)
          acc += __ldcg(p.partials + (static_cast<int64_t>(s) * B + j) * p.m_total + m);
        const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
        const __nv_bfloat16 lo = __float2bfloat16_rn(acc - __bfloat162float(hi));
        p.latent[static_cast<int64_t>(2 * j) * p.m_total + m] = hi;
        p.latent[static_cast<int64_t>(2 * j + 1) * p.m_total + m] = lo;
      }
      if (tid == 0) p.counters[m_tile] = 0;
    }
  }
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
  dim3 grid(m_tiles, p.mode == 0 ? p.splits : 1);
  mfa_qproj_kernel<<<grid, kGemmThreads, smem, stream>>>(tw, ta, p);
  return cudaGetLastError();
}

}  // namespace mfa
