// merge_kernel.cu -- log-sum-exp merge of attention results over disjoint key
// ranges (Flash-Decoding's combine, cited on the DeepSeek-V4 page's reference
// list): each part holds, per (sequence, head), the output normalised over its
// own range and that range's log-sum-exp; the merged output is
//
//     lse* = max_s lse_s,   w_s = exp(lse_s - lse*),
//     out  = sum_s w_s O_s / sum_s w_s,   lse = lse* + log sum_s w_s.
//
// This is the exchange step of a sequence whose cache is split across GPUs:
// each rank's decode-attention call returns (O, lse) over its key range, the
// parts are gathered, and this kernel merges them on the owner.
//
// HBM-bound: every part's 64 KB per sequence is read once. A CTA covers four
// heads of one sequence, a thread one float4 of head dims, so the whole grid
// streams (B x 16 CTAs) and each thread keeps eight parts' loads in flight.

#include "mfa_internal.h"
#include "sm100.cuh"

namespace mfa {

constexpr int kLseMergeHeads = 4;    // heads per CTA
constexpr int kLseMergeThreads = kLseMergeHeads * (kDim / 4);
constexpr int kLseMergeBatch = 8;    // parts whose loads are issued together

__global__ void __launch_bounds__(kLseMergeThreads) mfa_lse_merge_kernel(const LseMergeParams p) {
  constexpr int kCtasPerSeq = kHeads / kLseMergeHeads;
  constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
  const int b = blockIdx.x / kCtasPerSeq;
  const int h = (blockIdx.x % kCtasPerSeq) * kLseMergeHeads + threadIdx.x / (kDim / 4);
  const int d = (threadIdx.x % (kDim / 4)) * 4;
  const float* o_base = p.o_parts + b * p.o_sb + h * p.o_sh + d;
  const float* l_base = p.lse_parts + b * p.l_sb + h;

  // online merge in part order: running max m, weight sum l, weighted sums v
  float m = -INFINITY, l = 0.f;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < p.parts; s0 += kLseMergeBatch) {
    float e[kLseMergeBatch];
    float4 o[kLseMergeBatch];
#pragma unroll
    for (int k = 0; k < kLseMergeBatch; ++k) {
      const int s = s0 + k;
      e[k] = s < p.parts ? __ldcs(l_base + s * p.l_ss) : -INFINITY;
      o[k] = s < p.parts ? __ldcs(reinterpret_cast<const float4*>(o_base + s * p.o_ss))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    float mn = m;
#pragma unroll
    for (int k = 0; k < kLseMergeBatch; ++k) mn = fmaxf(mn, e[k]);
    if (mn == -INFINITY) continue;  // no weight so far
    const float c = ex2_approx((m - mn) * kLog2e);  // 0 while m is still -inf
    l *= c;
    v.x *= c;
    v.y *= c;
    v.z *= c;
    v.w *= c;
#pragma unroll
    for (int k = 0; k < kLseMergeBatch; ++k) {
      // a part with lse = -inf (an empty key range) has no weight, and its O
      // (whatever it holds) is not used
      if (e[k] > -INFINITY) {
        const float w = ex2_approx((e[k] - mn) * kLog2e);
        l += w;
        v.x += w * o[k].x;
        v.y += w * o[k].y;
        v.z += w * o[k].z;
        v.w += w * o[k].w;
      }
    }
    m = mn;
  }
  float lse = -INFINITY;
  if (m > -INFINITY) {
    const float inv = 1.f / l;
    v.x *= inv;
    v.y *= inv;
    v.z *= inv;
    v.w *= inv;
    lse = m + lg2_approx(l) * kLn2;
  }  // else every part is empty: zeros, lse = -inf (as an empty sequence)
  const int64_t off = b * p.out_sb + h * p.out_sh + d;
  if (p.out_f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(p.out) + off) = v;
  } else {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&lo);
    packed.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.out) + off) = packed;
  }
  if (p.lse_out && d == 0) p.lse_out[b * p.lse_sb + h] = lse;
}

cudaError_t launch_lse_merge(const LseMergeParams& p, cudaStream_t stream) {
  const unsigned ctas = static_cast<unsigned>(p.batch) * (kHeads / kLseMergeHeads);
  mfa_lse_merge_kernel<<<ctas, kLseMergeThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace mfa
