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
//   long_dyn_prep    one CTA per block, two passes over the hi rows: 1/|z_j|
//                    and the block sum s = sum_j u_j of the unit rows, then the
//                    row sums of the cosine matrix as u_i . s (the same sum,
//                    reassociated), so 1/(row sum + eps) is known before any
//                    Gram tile exists;
// and the hi-plane Gram itself, scaled to Gt and written as a split pair to
// the workspace, runs on tcgen05 (gram_tc_kernel in avey_mix_tc.cu).
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

// --------------------------------------------------------------- dynamic --

constexpr int kMaxMt = 1024;

// Per block: inv_n[j] = 1/max(|z_j|, 1e-12) of the hi rows, s = sum_j u_j with
// u_j = z_j inv_n[j], and inv_d[i] = 1/(u_i . s + eps): the row sum of the
// cosine matrix, sum_j u_i . u_j, taken as u_i . (sum_j u_j).  Two passes over
// the rows: the first gives each row's norm and adds its unit row into a
// per-warp partial of s held in registers (lane l owns features 8l + 256c ..
// +7); the second takes the dot products.  NC = ceil(mt / 256) chunks per lane.
template <int SL, int NC>
__global__ void __launch_bounds__(256) long_dyn_prep(const bf16 *__restrict__ zt, long long ld,
                                                     int mt, float eps, float *inv_n,
                                                     float *inv_d) {
  __shared__ float s_inv[SL];
  __shared__ float s_part[8][NC * 256];
  __shared__ float s_sum[NC * 256];
  const int blk = blockIdx.x;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bf16 *zb = zt + static_cast<long long>(blk) * SL * ld;
  float acc[NC][8];
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[c][q] = 0.f;
  for (int j = warp; j < SL; j += 8) {
    const bf16 *row = zb + static_cast<long long>(j) * ld;
    float v[NC][8];
    float ss = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int f = lane * 8 + 256 * c;
      uint4 q = make_uint4(0, 0, 0, 0);
      if (f < mt) q = *reinterpret_cast<const uint4 *>(row + f);
      const float2 a0 = unpack_bf16(q.x), a1 = unpack_bf16(q.y), a2 = unpack_bf16(q.z),
                   a3 = unpack_bf16(q.w);
      v[c][0] = a0.x; v[c][1] = a0.y; v[c][2] = a1.x; v[c][3] = a1.y;
      v[c][4] = a2.x; v[c][5] = a2.y; v[c][6] = a3.x; v[c][7] = a3.y;
#pragma unroll
      for (int q2 = 0; q2 < 8; ++q2) ss = fmaf(v[c][q2], v[c][q2], ss);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float inv = 1.f / fmaxf(sqrtf(ss), 1e-12f);
    if (lane == 0) {
      s_inv[j] = inv;
      inv_n[static_cast<long long>(blk) * SL + j] = inv;
    }
#pragma unroll
    for (int c = 0; c < NC; ++c)
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[c][q] = fmaf(v[c][q], inv, acc[c][q]);
  }
#pragma unroll
  for (int c = 0; c < NC; ++c)
#pragma unroll
    for (int q = 0; q < 8; ++q) s_part[warp][lane * 8 + 256 * c + q] = acc[c][q];
  __syncthreads();
  for (int f = tid; f < NC * 256; f += 256) {
    float t = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += s_part[w][f];
    s_sum[f] = t;
  }
  __syncthreads();
  for (int i = warp; i < SL; i += 8) {
    const bf16 *row = zb + static_cast<long long>(i) * ld;
    float dt = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const int f = lane * 8 + 256 * c;
      if (f >= mt) continue;
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
  switch ((mt + 255) / 256) {
    case 1: long_dyn_prep<SL, 1><<<blocks, 256, 0, s>>>(zt, ld, mt, eps, inv_n, inv_d); break;
    case 2: long_dyn_prep<SL, 2><<<blocks, 256, 0, s>>>(zt, ld, mt, eps, inv_n, inv_d); break;
    case 3: long_dyn_prep<SL, 3><<<blocks, 256, 0, s>>>(zt, ld, mt, eps, inv_n, inv_d); break;
    case 4: long_dyn_prep<SL, 4><<<blocks, 256, 0, s>>>(zt, ld, mt, eps, inv_n, inv_d); break;
    default:
      set_detail("long dynamic mix: m_t = %d above 1024", mt);
      return AVEY_ERR_UNSUPPORTED;
  }
  AVEY_CHECK_LAUNCH("long_dyn_prep", s);
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
