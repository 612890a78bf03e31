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
//                    1/(row sum + eps) is known before any Gram tile exists.
//   long_gram        one CTA per (block, 128 x 128 tile): the hi-plane Gram
//                    tile with mma.sync, scaled to Gt and written as a split
//                    pair to the workspace.
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

struct GramTile {
  static constexpr int TI = 128, FC = 64;
  static constexpr int CLD = FC + 8;               // bf16 (144 B)
  static constexpr int TBYTES = TI * CLD * 2;      // one 128-row chunk
  static constexpr int STAGES = 3;
  static constexpr int STAGE = 2 * TBYTES;         // i rows + j rows
  static constexpr int OLD = TI + 8;               // output staging row, bf16
  static constexpr int OBYTES = 2 * TI * OLD * 2;  // hi + lo
  static constexpr int SMEM = STAGES * STAGE > OBYTES ? STAGES * STAGE : OBYTES;
};

// Gt tile (rows i0.., columns j0..) of one block: the hi-plane Gram R_ij = z_i . z_j
// (mma.sync, fp32 accumulation) times inv_n[i] inv_n[j] inv_d[i], written as a
// split pair: gt[blk][i][j] (row-major SL x SL), lo plane at + gt_plane.
template <int SL>
__global__ void __launch_bounds__(256) long_gram(const bf16 *__restrict__ zt, long long ld, int mt,
                                                 const float *__restrict__ inv_n,
                                                 const float *__restrict__ inv_d, bf16 *gt,
                                                 long long gt_plane) {
  using C = GramTile;
  extern __shared__ __align__(16) uint8_t smem[];
  const int j0 = blockIdx.x * C::TI, i0 = blockIdx.y * C::TI, blk = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp / 4, wn = warp % 4;  // warp tile: 64 rows x 32 columns
  const bf16 *zb = zt + static_cast<long long>(blk) * SL * ld;
  const int nch = (mt + C::FC - 1) / C::FC;

  auto load = [&](int ch, int stg) {
    uint8_t *si = smem + stg * C::STAGE;
    uint8_t *sj = si + C::TBYTES;
    for (int e = tid; e < 2 * C::TI * (C::FC / 8); e += 256) {
      const int side = e / (C::TI * (C::FC / 8));
      const int r = e % (C::TI * (C::FC / 8));
      const int row = r / (C::FC / 8), cc = r % (C::FC / 8);
      const int f = ch * C::FC + cc * 8;
      const bool ok = f < mt;
      const bf16 *src = ok ? zb + static_cast<long long>((side ? j0 : i0) + row) * ld + f : zb;
      cp_async16(smem_u32((side ? sj : si) + (row * C::CLD + cc * 8) * 2), src, ok ? 16 : 0);
    }
    cp_async_commit();
  };

  float g[4][4][4] = {};
#pragma unroll
  for (int s = 0; s < C::STAGES - 1; ++s) {
    if (s < nch)
      load(s, s);
    else
      cp_async_commit();
  }
#pragma unroll 1
  for (int ch = 0; ch < nch; ++ch) {
    cp_async_wait<C::STAGES - 2>();
    __syncthreads();
    if (ch + C::STAGES - 1 < nch)
      load(ch + C::STAGES - 1, (ch + C::STAGES - 1) % C::STAGES);
    else
      cp_async_commit();
    const uint8_t *si = smem + (ch % C::STAGES) * C::STAGE;
    const uint8_t *sj = si + C::TBYTES;
#pragma unroll
    for (int kk = 0; kk < C::FC; kk += 16) {
      uint32_t af[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = wm * 64 + i * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldsm_x4(smem_u32(si + (row * C::CLD + kk + (lane >> 4) * 8) * 2), af[i][0], af[i][1],
                af[i][2], af[i][3]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        uint32_t b0, b1;
        const int jrow = wn * 32 + j * 8 + (lane & 7);
        ldsm_x2(smem_u32(sj + (jrow * C::CLD + kk + ((lane >> 3) & 1) * 8) * 2), b0, b1);
        const uint32_t bb[2] = {b0, b1};
#pragma unroll
        for (int i = 0; i < 4; ++i) mma16816(g[i][j], af[i], bb);
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  const float *nb = inv_n + static_cast<long long>(blk) * SL;
  const float *db = inv_d + static_cast<long long>(blk) * SL;
  uint8_t *oh = smem;
  uint8_t *ol = smem + C::TI * C::OLD * 2;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int row = wm * 64 + i * 16 + (lane >> 2) + hh * 8;
      const float ri = nb[i0 + row] * db[i0 + row];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = wn * 32 + j * 8 + (lane & 3) * 2;
        const float v0 = g[i][j][2 * hh] * ri * nb[j0 + col];
        const float v1 = g[i][j][2 * hh + 1] * ri * nb[j0 + col + 1];
        uint32_t hi, lo;
        split_pack(v0, v1, hi, lo);
        *reinterpret_cast<uint32_t *>(oh + (row * C::OLD + col) * 2) = hi;
        *reinterpret_cast<uint32_t *>(ol + (row * C::OLD + col) * 2) = lo;
      }
    }
  __syncthreads();
  bf16 *gb = gt + static_cast<long long>(blk) * SL * SL;
  for (int e = tid; e < C::TI * (C::TI / 8); e += 256) {
    const int row = e / (C::TI / 8), cc = e % (C::TI / 8);
    bf16 *dst = gb + static_cast<long long>(i0 + row) * SL + j0 + cc * 8;
    *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(oh + (row * C::OLD + cc * 8) * 2);
    *reinterpret_cast<uint4 *>(dst + gt_plane) =
        *reinterpret_cast<const uint4 *>(ol + (row * C::OLD + cc * 8) * 2);
  }
}

template <typename K>
avey_status set_smem_long(K kern, int bytes, const char *name) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    set_detail("%s: cudaFuncSetAttribute: %s", name, cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  return AVEY_OK;
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
  auto gk = long_gram<SL>;
  avey_status st = set_smem_long(gk, GramTile::SMEM, "long_gram");
  if (st != AVEY_OK) return st;
  gk<<<dim3(SL / GramTile::TI, SL / GramTile::TI, blocks), 256, GramTile::SMEM, s>>>(
      zt, ld, mt, inv_n, inv_d, gt, gt_plane);
  AVEY_CHECK_LAUNCH("long_gram");
  return AVEY_OK;
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
