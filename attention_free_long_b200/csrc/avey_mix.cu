// avey_mix.cu -- the contextualizer of a neural-processor layer, applied per
// split block of S tokens (papernotes 关键设计 2 and 3; paperlayer summary §4.2):
//   static:   c = V Z_t                      (learned S x S map, signed)
//   dynamic:  G_ij = N(z_i).N(z_j);  Gt_ij = G_ij / (sum_j G_ij + eps)  (eq. 6)
//             c = Gt Z_t
// Identity activation, no bias.
//
// The bf16 mixes (Z_t an activation split pair) run on tcgen05 in
// avey_mix_dyn.cu.  This file holds the fp32 path (plain SIMT kernels) and the
// C ABI entry points of both mixes.
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

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

}  // namespace

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
