// avey_mix.cu -- the contextualizer of a neural-processor layer, applied per
// split block of S tokens (papernotes 关键设计 2 and 3; paperlayer summary §4.2):
//   static:   c = V Z_t                      (learned S x S map, signed)
//   dynamic:  G_ij = N(z_i).N(z_j);  Gt_ij = G_ij / (sum_j G_ij + eps)  (eq. 6)
//             c = Gt Z_t
// Identity activation, no bias.
//
// bf16 path: Z_t is an activation split pair (hi, lo bf16 planes).  The
// static mix is bound by HBM (read Z_t, write c, 8 bytes per element each way):
//   static_mix_x2   one CTA per (block, feature slab); V and both planes of
//                   the slab in shared memory; c = V Z_hi + V Z_lo with
//                   mma.sync; written back in place as a split pair.
// The bf16 dynamic (and coupled causal) mix runs on tcgen05 in
// avey_mix_dyn.cu.  fp32 path: plain SIMT kernels, and the C ABI entry points
// of both mixes.
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

// ---------------------------------------------------------------- static --

template <int S>
struct StaticTile {
  static constexpr int WM = S >= 32 ? 32 : 16;
  static constexpr int WARPS_M = S / WM;
  static constexpr int WARPS_N = 8 / WARPS_M;
  static constexpr int WN = 32;
  static constexpr int NS = WN * WARPS_N;
  static constexpr int MI = WM / 16, NI = WN / 8;
  static constexpr int ZLD = NS + 8, VLD = S + 8;
  static constexpr int ZBYTES = S * ZLD * 2, VBYTES = S * VLD * 2;
  static constexpr int SMEM = VBYTES + 2 * ZBYTES;
};

template <int S>
__global__ void __launch_bounds__(256) static_mix_x2(const bf16 *__restrict__ V, const bf16 *zt,
                                                     long long ld, int mt, long long plane,
                                                     bf16 *out, long long ld_out,
                                                     long long plane_out) {
  using C = StaticTile<S>;
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t *vs = smem;
  uint8_t *zh = smem + C::VBYTES;
  uint8_t *zl = zh + C::ZBYTES;
  const int slab = blockIdx.x, blk = blockIdx.y;
  const int f0 = slab * C::NS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp / C::WARPS_N, wn = warp % C::WARPS_N;
  const bf16 *zbase = zt + static_cast<long long>(blk) * S * ld;
  bf16 *obase = out + static_cast<long long>(blk) * S * ld_out;

  for (int e = tid; e < S * (S / 8); e += 256) {
    const int row = e / (S / 8), cc = e % (S / 8);
    cp_async16(smem_u32(vs + (row * C::VLD + cc * 8) * 2), V + row * S + cc * 8, 16);
  }
  for (int e = tid; e < S * (C::NS / 8); e += 256) {
    const int row = e / (C::NS / 8), cc = e % (C::NS / 8);
    const int f = f0 + cc * 8;
    const bool ok = f < mt;
    const bf16 *src = ok ? zbase + row * ld + f : zbase;
    cp_async16(smem_u32(zh + (row * C::ZLD + cc * 8) * 2), src, ok ? 16 : 0);
    cp_async16(smem_u32(zl + (row * C::ZLD + cc * 8) * 2), ok ? src + plane : zbase, ok ? 16 : 0);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();

  float acc[C::MI][C::NI][4] = {};
#pragma unroll
  for (int kk = 0; kk < S; kk += 16) {
    uint32_t af[C::MI][4];
#pragma unroll
    for (int i = 0; i < C::MI; ++i) {
      const int row = wm * C::WM + i * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
      ldsm_x4(smem_u32(vs + (row * C::VLD + kk + (lane >> 4) * 8) * 2), af[i][0], af[i][1], af[i][2],
              af[i][3]);
    }
#pragma unroll
    for (int j = 0; j < C::NI; j += 2) {
      const int krow = kk + (lane & 7) + ((lane >> 3) & 1) * 8;
      const int ncol = wn * C::WN + j * 8 + (lane >> 4) * 8;
#pragma unroll
      for (int pl = 0; pl < 2; ++pl) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32((pl ? zl : zh) + (krow * C::ZLD + ncol) * 2), b0, b1, b2, b3);
        const uint32_t bA[2] = {b0, b1}, bB[2] = {b2, b3};
#pragma unroll
        for (int i = 0; i < C::MI; ++i) {
          mma16816(acc[i][j], af[i], bA);
          mma16816(acc[i][j + 1], af[i], bB);
        }
      }
    }
  }
  // c as a split pair, staged over the (now consumed) input slab, then written
  // back with coalesced 16-byte stores.
  __syncthreads();
#pragma unroll
  for (int i = 0; i < C::MI; ++i)
#pragma unroll
    for (int j = 0; j < C::NI; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = wm * C::WM + i * 16 + (lane >> 2) + h * 8;
        const int fl = wn * C::WN + j * 8 + (lane & 3) * 2;
        uint32_t hi, lo;
        split_pack(acc[i][j][2 * h], acc[i][j][2 * h + 1], hi, lo);
        *reinterpret_cast<uint32_t *>(zh + (row * C::ZLD + fl) * 2) = hi;
        *reinterpret_cast<uint32_t *>(zl + (row * C::ZLD + fl) * 2) = lo;
      }
  __syncthreads();
  for (int e = tid; e < S * (C::NS / 8); e += 256) {
    const int row = e / (C::NS / 8), cc = e % (C::NS / 8);
    const int f = f0 + cc * 8;
    if (f >= mt) continue;
    bf16 *dst = obase + row * ld_out + f;
    *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(zh + (row * C::ZLD + cc * 8) * 2);
    *reinterpret_cast<uint4 *>(dst + plane_out) =
        *reinterpret_cast<const uint4 *>(zl + (row * C::ZLD + cc * 8) * 2);
  }
}

// ------------------------------------------------------------------ fp32 --

template <int S>
__global__ void __launch_bounds__(256) static_mix_f32(const float *__restrict__ V, const float *zt,
                                                      long long ld_zt, float *out,
                                                      long long ld_out, int mt) {
  constexpr int NSL = 64;
  __shared__ float vs[S][S];
  __shared__ float zs[S][NSL];
  const int slab = blockIdx.x, blk = blockIdx.y, tid = threadIdx.x;
  const int f0 = slab * NSL;
  const float *zb = zt + static_cast<long long>(blk) * S * ld_zt;
  float *ob = out + static_cast<long long>(blk) * S * ld_out;
  for (int e = tid; e < S * S; e += 256) vs[e / S][e % S] = V[e];
  for (int e = tid; e < S * NSL; e += 256) {
    const int r = e / NSL, c = e % NSL;
    zs[r][c] = (f0 + c < mt) ? zb[r * ld_zt + f0 + c] : 0.f;
  }
  __syncthreads();
  for (int e = tid; e < S * NSL; e += 256) {
    const int i = e / NSL, c = e % NSL;
    if (f0 + c >= mt) continue;
    float s = 0.f;
    for (int j = 0; j < S; ++j) s = fmaf(vs[i][j], zs[j][c], s);
    ob[i * ld_out + f0 + c] = s;
  }
}

template <int S, bool COUPLED>
__global__ void __launch_bounds__(256) dynamic_mix_f32(const float *zt, long long ld_zt,
                                                       float *out, long long ld_out, int mt,
                                                       float eps, const float *__restrict__ V) {
  constexpr int NSL = 64;
  __shared__ float Gt[S][S + 1];
  __shared__ float nf[S];
  __shared__ float zs[S][NSL];
  const int blk = blockIdx.x, tid = threadIdx.x;
  const float *zb = zt + static_cast<long long>(blk) * S * ld_zt;
  float *ob = out + static_cast<long long>(blk) * S * ld_out;
  if (tid < S) {
    float ss = 0.f;
    for (int f = 0; f < mt; ++f) ss = fmaf(zb[tid * ld_zt + f], zb[tid * ld_zt + f], ss);
    nf[tid] = fmaxf(sqrtf(ss), 1e-12f);
  }
  __syncthreads();
  for (int e = tid; e < S * S; e += 256) {
    const int i = e / S, j = e % S;
    float s = 0.f;
    for (int f = 0; f < mt; ++f) s = fmaf(zb[i * ld_zt + f], zb[j * ld_zt + f], s);
    Gt[i][j] = s / (nf[i] * nf[j]);
  }
  __syncthreads();
  if (tid < S) {
    if constexpr (COUPLED) {
      for (int j = 0; j < S; ++j) Gt[tid][j] = j <= tid ? V[tid * S + j] * Gt[tid][j] : 0.f;
    } else {
      float rs = 0.f;
      for (int j = 0; j < S; ++j) rs += Gt[tid][j];
      const float den = rs + eps;
      for (int j = 0; j < S; ++j) Gt[tid][j] = Gt[tid][j] / den;
    }
  }
  __syncthreads();
  // c = Gt Z_t, slab by slab; every slab is read into shared memory before
  // its outputs are written, so out may alias zt.
  for (int f0 = 0; f0 < mt; f0 += NSL) {
    for (int e = tid; e < S * NSL; e += 256) {
      const int r = e / NSL, c = e % NSL;
      zs[r][c] = (f0 + c < mt) ? zb[r * ld_zt + f0 + c] : 0.f;
    }
    __syncthreads();
    for (int e = tid; e < S * NSL; e += 256) {
      const int i = e / NSL, c = e % NSL;
      if (f0 + c >= mt) continue;
      float s = 0.f;
      for (int j = 0; j < S; ++j) s = fmaf(Gt[i][j], zs[j][c], s);
      ob[i * ld_out + f0 + c] = s;
    }
    __syncthreads();
  }
}

template <typename K>
avey_status set_smem(K kern, int bytes, const char *name) {
  if (bytes <= 48 * 1024) return AVEY_OK;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) {
    set_detail("%s: %s", name, cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  return AVEY_OK;
}

template <int S>
avey_status run_static_x2(const bf16 *V, const bf16 *zt, int64_t ld, int blocks, int mt,
                          int64_t plane, bf16 *out, int64_t ld_out, int64_t plane_out,
                          cudaStream_t s) {
  using C = StaticTile<S>;
  if (avey_status st = set_smem(static_mix_x2<S>, C::SMEM, "static_mix_x2")) return st;
  const dim3 grid((mt + C::NS - 1) / C::NS, blocks);
  static_mix_x2<S><<<grid, 256, C::SMEM, s>>>(V, zt, ld, mt, plane, out, ld_out, plane_out);
  AVEY_CHECK_LAUNCH("static_mix_x2", s);
  return AVEY_OK;
}

}  // namespace

avey_status launch_static_mix_x2(const bf16 *V, const bf16 *zt, int64_t ld, int blocks, int S,
                                 int mt, int64_t plane, bf16 *out, int64_t ld_out,
                                 int64_t plane_out, cudaStream_t s) {
  switch (S) {
    case 16: return run_static_x2<16>(V, zt, ld, blocks, mt, plane, out, ld_out, plane_out, s);
    case 32: return run_static_x2<32>(V, zt, ld, blocks, mt, plane, out, ld_out, plane_out, s);
    case 64: return run_static_x2<64>(V, zt, ld, blocks, mt, plane, out, ld_out, plane_out, s);
    case 128: return run_static_x2<128>(V, zt, ld, blocks, mt, plane, out, ld_out, plane_out, s);
  }
  set_detail("static mix: S=%d unsupported", S);
  return AVEY_ERR_UNSUPPORTED;
}

avey_status launch_static_mix_f32(const float *V, const float *zt, int64_t ld_zt, float *out,
                                  int64_t ld_out, int blocks, int S, int mt, cudaStream_t s) {
  const dim3 grid((mt + 63) / 64, blocks);
  switch (S) {
#define AVEY_SF(SS) \
  case SS: static_mix_f32<SS><<<grid, 256, 0, s>>>(V, zt, ld_zt, out, ld_out, mt); break;
    AVEY_SF(1) AVEY_SF(2) AVEY_SF(4) AVEY_SF(8) AVEY_SF(16) AVEY_SF(32) AVEY_SF(64)
#undef AVEY_SF
    default: set_detail("static mix (F32): S=%d unsupported", S); return AVEY_ERR_UNSUPPORTED;
  }
  AVEY_CHECK_LAUNCH("static_mix_f32", s);
  return AVEY_OK;
}

avey_status launch_dynamic_mix_f32(const float *zt, int64_t ld_zt, float *out, int64_t ld_out,
                                   int blocks, int S, int mt, float eps, cudaStream_t s) {
  switch (S) {
#define AVEY_DF(SS) \
  case SS: dynamic_mix_f32<SS, false><<<blocks, 256, 0, s>>>(zt, ld_zt, out, ld_out, mt, eps, nullptr); break;
    AVEY_DF(1) AVEY_DF(2) AVEY_DF(4) AVEY_DF(8) AVEY_DF(16) AVEY_DF(32) AVEY_DF(64)
#undef AVEY_DF
    default: set_detail("dynamic mix (F32): S=%d unsupported", S); return AVEY_ERR_UNSUPPORTED;
  }
  AVEY_CHECK_LAUNCH("dynamic_mix_f32", s);
  return AVEY_OK;
}

avey_status launch_coupled_mix_f32(const float *V, const float *zt, int64_t ld_zt, float *out,
                                   int64_t ld_out, int blocks, int S, int mt, cudaStream_t s) {
  switch (S) {
#define AVEY_CF(SS) \
  case SS: dynamic_mix_f32<SS, true><<<blocks, 256, 0, s>>>(zt, ld_zt, out, ld_out, mt, 0.f, V); break;
    AVEY_CF(1) AVEY_CF(2) AVEY_CF(4) AVEY_CF(8) AVEY_CF(16) AVEY_CF(32) AVEY_CF(64)
#undef AVEY_CF
    default: set_detail("coupled mix (F32): S=%d unsupported", S); return AVEY_ERR_UNSUPPORTED;
  }
  AVEY_CHECK_LAUNCH("coupled_mix_f32", s);
  return AVEY_OK;
}

}  // namespace avey

using namespace avey;

extern "C" avey_status avey_static_mix(const void *V, const void *zt, int64_t ld_zt, avey_dtype dt,
                                       int blocks, int S, int mt, void *out, int64_t ld_out,
                                       avey_stream_t stream) {
  AVEY_REQUIRE(dt == AVEY_F32 || dt == AVEY_BF16X2, AVEY_ERR_UNSUPPORTED,
               "avey_static_mix: dtype %d unsupported (F32 or BF16X2)", int(dt));
  AVEY_REQUIRE(V && zt && out, AVEY_ERR_INVALID_ARG, "avey_static_mix: null pointer");
  AVEY_REQUIRE(blocks >= 0 && S >= 1 && mt >= 1 && ld_zt >= mt && ld_out >= mt,
               AVEY_ERR_INVALID_ARG, "avey_static_mix: bad sizes");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (blocks == 0) return AVEY_OK;
  const char *zb = static_cast<const char *>(zt);
  const char *obp = static_cast<const char *>(out);
  const size_t es = dt == AVEY_F32 ? 4 : 2;
  const size_t planes = dt == AVEY_BF16X2 ? 2 : 1;
  const size_t zspan = static_cast<size_t>(blocks) * S * ld_zt * es * planes;
  const size_t ospan = static_cast<size_t>(blocks) * S * ld_out * es * planes;
  const bool same = zt == out && ld_zt == ld_out;
  const bool overlap = !same && zb < obp + ospan && obp < zb + zspan;
  AVEY_REQUIRE(!overlap, AVEY_ERR_INVALID_ARG,
               "avey_static_mix: out overlaps zt without aliasing it exactly");
  if (dt == AVEY_BF16X2) {
    AVEY_REQUIRE(S == 16 || S == 32 || S == 64 || S == 128, AVEY_ERR_UNSUPPORTED,
                 "avey_static_mix(BF16X2): S=%d unsupported (16, 32, 64 or 128)", S);
    AVEY_REQUIRE(mt % 8 == 0 && ld_zt % 8 == 0 && ld_out % 8 == 0 && aligned16(zt) &&
                     aligned16(out) && aligned16(V),
                 AVEY_ERR_INVALID_ARG,
                 "avey_static_mix(BF16X2): mt and ld must be multiples of 8, pointers 16-byte aligned");
    const int64_t pz = static_cast<int64_t>(blocks) * S * ld_zt;
    const int64_t po = static_cast<int64_t>(blocks) * S * ld_out;
    return launch_static_mix_x2(static_cast<const bf16 *>(V), static_cast<const bf16 *>(zt), ld_zt,
                                blocks, S, mt, pz, static_cast<bf16 *>(out), ld_out, po, s);
  }
  AVEY_REQUIRE(S <= 64 && (S & (S - 1)) == 0, AVEY_ERR_UNSUPPORTED,
               "avey_static_mix(F32): S=%d unsupported (power of two <= 64)", S);
  return launch_static_mix_f32(static_cast<const float *>(V), static_cast<const float *>(zt), ld_zt,
                               static_cast<float *>(out), ld_out, blocks, S, mt, s);
}

extern "C" avey_status avey_dynamic_mix(const void *zt, int64_t ld_zt, avey_dtype dt, int blocks,
                                        int S, int mt, float eps, void *out, int64_t ld_out,
                                        avey_stream_t stream) {
  AVEY_REQUIRE(dt == AVEY_F32 || dt == AVEY_BF16X2, AVEY_ERR_UNSUPPORTED,
               "avey_dynamic_mix: dtype %d unsupported (F32 or BF16X2)", int(dt));
  AVEY_REQUIRE(zt && out, AVEY_ERR_INVALID_ARG, "avey_dynamic_mix: null pointer");
  AVEY_REQUIRE(blocks >= 0 && S >= 1 && mt >= 1 && ld_zt >= mt && ld_out >= mt && eps >= 0.f,
               AVEY_ERR_INVALID_ARG, "avey_dynamic_mix: bad sizes");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (blocks == 0) return AVEY_OK;
  const char *zb = static_cast<const char *>(zt);
  const char *obp = static_cast<const char *>(out);
  const size_t es = dt == AVEY_F32 ? 4 : 2;
  const size_t zspan = static_cast<size_t>(blocks) * S * ld_zt * es;
  const size_t ospan = static_cast<size_t>(blocks) * S * ld_out * es;
  const bool same = zt == out && ld_zt == ld_out;
  const bool overlap = !same && zb < obp + ospan * (dt == AVEY_BF16X2 ? 2 : 1) &&
                       obp < zb + zspan * (dt == AVEY_BF16X2 ? 2 : 1);
  AVEY_REQUIRE(!overlap, AVEY_ERR_INVALID_ARG,
               "avey_dynamic_mix: out overlaps zt without aliasing it exactly");
  if (dt == AVEY_BF16X2) {
    AVEY_REQUIRE(S == 16 || S == 32 || S == 64 || S == 128, AVEY_ERR_UNSUPPORTED,
                 "avey_dynamic_mix(BF16X2): S=%d unsupported (16, 32, 64 or 128)", S);
    AVEY_REQUIRE(mt % 8 == 0 && ld_zt % 8 == 0 && ld_out % 8 == 0 && aligned16(zt) && aligned16(out),
                 AVEY_ERR_INVALID_ARG,
                 "avey_dynamic_mix(BF16X2): mt and ld must be multiples of 8, pointers 16-byte aligned");
    const int64_t pz = static_cast<int64_t>(blocks) * S * ld_zt;
    const int64_t po = static_cast<int64_t>(blocks) * S * ld_out;
    return launch_dynamic_mix_x2(static_cast<const bf16 *>(zt), ld_zt, pz, static_cast<bf16 *>(out),
                                 ld_out, po, blocks, S, mt, eps, s);
  }
  AVEY_REQUIRE(S <= 64 && (S & (S - 1)) == 0, AVEY_ERR_UNSUPPORTED,
               "avey_dynamic_mix(F32): S=%d unsupported (power of two <= 64)", S);
  return launch_dynamic_mix_f32(static_cast<const float *>(zt), ld_zt, static_cast<float *>(out),
                                ld_out, blocks, S, mt, eps, s);
}
