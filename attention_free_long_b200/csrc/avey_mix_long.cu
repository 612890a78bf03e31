// avey_mix_long.cu -- the contextualizer over long token blocks (256 or 512
// tokens), used by the processor without neural compression: each target
// split is processed together with its k retrieved splits, so the mix runs
// over (k+1)S tokens (Avey-B paperlayer summary §4.3, the ablation behind the
// 4.37x throughput figure; papernotes 关键设计 2-3 for the mixes themselves):
//   static:   c = V Z_t,  V of size (k+1)S x (k+1)S
//   dynamic:  Gt_ij = N(z_i).N(z_j) / (sum_j N(z_i).N(z_j) + eps),  c = Gt Z_t
// Z_t is the activation split pair (hi, lo bf16 planes).
//
// At SL = 512 the mix is a real contraction (2 SL FLOP per output element)
// whose per-block operand (V or Gt, SL x SL) no longer fits in shared memory
// next to the activations; c = A Z_t itself runs on tcgen05 (avey_mix_tc.cu).
// This file builds the dynamic A, Gt, per block:
//   long_dyn_prep    one CTA per block: 1/|z_j| of the hi rows, the block sum
//                    s = sum_j u_j of the unit rows, and the row sums of the
//                    cosine matrix as u_i . s (the same sum, reassociated), so
//                    1/(row sum + eps) is known before any Gram tile exists;
// and the hi-plane Gram itself, scaled to Gt and written as a split pair to
// the workspace, runs on tcgen05 (gram_tc_kernel in avey_mix_tc.cu).
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

// --------------------------------------------------------------- dynamic --

constexpr int kMaxMt = 4096;

// Per block: inv_n[j] = 1/max(|z_j|, 1e-12) of the hi rows, s = sum_j u_j with
// u_j = z_j inv_n[j], and inv_d[i] = 1/(u_i . s + eps): the row sum of the
// cosine matrix, sum_j u_i . u_j, taken as u_i . (sum_j u_j).
template <int SL>
__global__ void __launch_bounds__(256) long_dyn_prep(const bf16 *__restrict__ zt, long long ld,
                                                     int mt, float eps, float *inv_n,
                                                     float *inv_d) {
  __shared__ float s_inv[SL];
  __shared__ float s_sum[kMaxMt];
  const int blk = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bf16 *zb = zt + static_cast<long long>(blk) * SL * ld;
  for (int j = warp; j < SL; j += 8) {
    const bf16 *row = zb + static_cast<long long>(j) * ld;
    float ss = 0.f;
    for (int f = lane * 8; f < mt; f += 256) {
      const uint4 q = *reinterpret_cast<const uint4 *>(row + f);
      const float2 v0 = unpack_bf16(q.x), v1 = unpack_bf16(q.y), v2 = unpack_bf16(q.z),
                   v3 = unpack_bf16(q.w);
      ss = fmaf(v0.x, v0.x, fmaf(v0.y, v0.y, ss));
      ss = fmaf(v1.x, v1.x, fmaf(v1.y, v1.y, ss));
      ss = fmaf(v2.x, v2.x, fmaf(v2.y, v2.y, ss));
      ss = fmaf(v3.x, v3.x, fmaf(v3.y, v3.y, ss));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    if (lane == 0) {
      const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
      s_inv[j] = inv;
      inv_n[static_cast<long long>(blk) * SL + j] = inv;
    }
  }
  __syncthreads();
  for (int f = 2 * tid; f < mt; f += 512) {
    float a = 0.f, b = 0.f;
    for (int j = 0; j < SL; ++j) {
      const float2 v = unpack_bf16(*reinterpret_cast<const uint32_t *>(zb + static_cast<long long>(j) * ld + f));
      a = fmaf(v.x, s_inv[j], a);
      b = fmaf(v.y, s_inv[j], b);
    }
    s_sum[f] = a;
    s_sum[f + 1] = b;
  }
  __syncthreads();
  for (int i = warp; i < SL; i += 8) {
    const bf16 *row = zb + static_cast<long long>(i) * ld;
    float dt = 0.f;
    for (int f = lane * 8; f < mt; f += 256) {
      const uint4 q = *reinterpret_cast<const uint4 *>(row + f);
      const float2 v0 = unpack_bf16(q.x), v1 = unpack_bf16(q.y), v2 = unpack_bf16(q.z),
                   v3 = unpack_bf16(q.w);
      dt = fmaf(v0.x, s_sum[f], fmaf(v0.y, s_sum[f + 1], dt));
      dt = fmaf(v1.x, s_sum[f + 2], fmaf(v1.y, s_sum[f + 3], dt));
      dt = fmaf(v2.x, s_sum[f + 4], fmaf(v2.y, s_sum[f + 5], dt));
      dt = fmaf(v3.x, s_sum[f + 6], fmaf(v3.y, s_sum[f + 7], dt));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) dt += __shfl_xor_sync(0xffffffffu, dt, off);
    if (lane == 0) inv_d[static_cast<long long>(blk) * SL + i] = 1.f / (dt * s_inv[i] + eps);
  }
}

template <int SL>
avey_status run_dynamic_gt(const bf16 *zt, int64_t ld, int blocks, int mt, float eps, void *ws,
                           cudaStream_t s) {
  const long long gt_plane = static_cast<long long>(blocks) * SL * SL;
  bf16 *gt = static_cast<bf16 *>(ws);
  float *inv_n = reinterpret_cast<float *>(gt + 2 * gt_plane);
  float *inv_d = inv_n + static_cast<long long>(blocks) * SL;
  long_dyn_prep<SL><<<blocks, 256, 0, s>>>(zt, ld, mt, eps, inv_n, inv_d);
  AVEY_CHECK_LAUNCH("long_dyn_prep");
  return launch_long_gram_tc(zt, ld, blocks, SL, mt, inv_n, inv_d, gt, s);
}

}  // namespace

size_t long_dynamic_ws_bytes(int blocks, int SL) {
  if (SL != 256 && SL != 512) return 0;
  return static_cast<size_t>(blocks) * SL * SL * 4 + static_cast<size_t>(blocks) * SL * 8;
}

avey_status launch_long_dynamic_gt(const bf16 *zt, int64_t ld, int blocks, int SL, int mt, float eps,
                                   void *ws, cudaStream_t s) {
  AVEY_REQUIRE(mt % 8 == 0 && ld % 8 == 0 && mt <= kMaxMt, AVEY_ERR_INVALID_ARG,
               "long dynamic mix: mt (<= %d) and ld must be multiples of 8", kMaxMt);
  AVEY_REQUIRE((reinterpret_cast<uintptr_t>(ws) & 15) == 0, AVEY_ERR_INVALID_ARG,
               "long dynamic mix: workspace must be 16-byte aligned");
  AVEY_REQUIRE(blocks >= 1 && blocks <= 65535, AVEY_ERR_UNSUPPORTED,
               "long dynamic mix: %d blocks (1 .. 65535)", blocks);
  switch (SL) {
    case 256: return run_dynamic_gt<256>(zt, ld, blocks, mt, eps, ws, s);
    case 512: return run_dynamic_gt<512>(zt, ld, blocks, mt, eps, ws, s);
    default: set_detail("long dynamic mix: block of %d tokens unsupported", SL); return AVEY_ERR_UNSUPPORTED;
  }
}

}  // namespace avey
