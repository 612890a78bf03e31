// avey_context.cu -- the uncompressed context of every split, for the
// processor without neural compression (Avey-B paperlayer summary §4.3: the
// ablation that the 4.37x throughput figure compares against; papernotes
// 关键设计 4 for the context itself, the compressor's input of eq. 8):
//   ctx(b, t) = [X_t ; w_1 X_c1 ; ... ; w_k X_ck]     ((k+1)S x d, rank order)
// The target block is unweighted; a candidate of -1 and the pad rows of a
// ragged last split give zero rows.  HBM-bound gather: every thread moves 8
// consecutive features of one output row (one 16-byte load of bf16 X), writes
// them as fp32 and, for bf16 inputs, as the activation split pair that the
// first layer's enricher reads.
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

template <bool BF16_IN>
__global__ void __launch_bounds__(256)
    context_rows(const void *__restrict__ x, int N, int d, int S, int k, int n,
                 const int32_t *__restrict__ idx, const float *__restrict__ w, float *out,
                 bf16 *ohi, bf16 *olo, long long units, int *status) {
  const int cpr = d / 8;  // 8-feature chunks per row
  const int L = (k + 1) * S;
  for (long long u = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; u < units;
       u += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long row = u / cpr;
    const int cc = static_cast<int>(u - row * cpr);
    const long long seg = row / L;  // b * n + t
    const int rin = static_cast<int>(row - seg * L);
    const int r = rin / S, j = rin - r * S;
    const int b = static_cast<int>(seg / n), t = static_cast<int>(seg - static_cast<long long>(b) * n);
    int c = t;
    float wr = 1.f;
    if (r > 0) {
      c = __ldg(idx + seg * k + (r - 1));
      wr = __ldg(w + seg * k + (r - 1));
      if (c < -1 || c >= n) {
        record_status(status, AVEY_ERR_DEVICE_BOUNDS);
        c = -1;
      }
    }
    const long long tok = static_cast<long long>(c) * S + j;
    const bool valid = c >= 0 && tok < N;
    float v[8];
    if (BF16_IN) {
      uint4 q = make_uint4(0, 0, 0, 0);
      if (valid)
        q = __ldg(reinterpret_cast<const uint4 *>(static_cast<const bf16 *>(x) +
                                                  (static_cast<long long>(b) * N + tok) * d + cc * 8));
      const float2 a0 = unpack_bf16(q.x), a1 = unpack_bf16(q.y), a2 = unpack_bf16(q.z),
                   a3 = unpack_bf16(q.w);
      v[0] = a0.x; v[1] = a0.y; v[2] = a1.x; v[3] = a1.y;
      v[4] = a2.x; v[5] = a2.y; v[6] = a3.x; v[7] = a3.y;
    } else {
      float4 p0 = make_float4(0.f, 0.f, 0.f, 0.f), p1 = p0;
      if (valid) {
        const float4 *src = reinterpret_cast<const float4 *>(
            static_cast<const float *>(x) + (static_cast<long long>(b) * N + tok) * d + cc * 8);
        p0 = __ldg(src);
        p1 = __ldg(src + 1);
      }
      v[0] = p0.x; v[1] = p0.y; v[2] = p0.z; v[3] = p0.w;
      v[4] = p1.x; v[5] = p1.y; v[6] = p1.z; v[7] = p1.w;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) v[q] *= wr;
    float4 *dst = reinterpret_cast<float4 *>(out + row * d + cc * 8);
    dst[0] = make_float4(v[0], v[1], v[2], v[3]);
    dst[1] = make_float4(v[4], v[5], v[6], v[7]);
    if (ohi) {
      uint4 h, l;
      split_pack(v[0], v[1], h.x, l.x);
      split_pack(v[2], v[3], h.y, l.y);
      split_pack(v[4], v[5], h.z, l.z);
      split_pack(v[6], v[7], h.w, l.w);
      *reinterpret_cast<uint4 *>(ohi + row * d + cc * 8) = h;
      *reinterpret_cast<uint4 *>(olo + row * d + cc * 8) = l;
    }
  }
}

}  // namespace
}  // namespace avey

using namespace avey;

extern "C" avey_status avey_context(const void *x, avey_dtype dt, int B, int N, int d, int S, int k,
                                    const int32_t *idx, const float *w, float *out, void *out_lowp,
                                    avey_stream_t stream) {
  AVEY_REQUIRE(dt == AVEY_F32 || dt == AVEY_BF16, AVEY_ERR_UNSUPPORTED,
               "avey_context: dtype %d unsupported (F32 or BF16)", int(dt));
  AVEY_REQUIRE(x && idx && w && out, AVEY_ERR_INVALID_ARG, "avey_context: null pointer");
  AVEY_REQUIRE(B >= 1 && N >= 1 && d >= 1 && S >= 1 && k >= 1, AVEY_ERR_INVALID_ARG,
               "avey_context: sizes must be >= 1 (B=%d N=%d d=%d S=%d k=%d)", B, N, d, S, k);
  AVEY_REQUIRE(d % 8 == 0, AVEY_ERR_INVALID_ARG, "avey_context: d=%d must be a multiple of 8", d);
  AVEY_REQUIRE(k <= 32, AVEY_ERR_UNSUPPORTED, "avey_context: k=%d > 32", k);
  AVEY_REQUIRE(aligned16(x) && aligned16(out) && (!out_lowp || aligned16(out_lowp)),
               AVEY_ERR_INVALID_ARG, "avey_context: pointers must be 16-byte aligned");
  const long long n = (N + S - 1) / S;
  const long long rows = static_cast<long long>(B) * n * (k + 1) * S;
  AVEY_REQUIRE(rows * d < (1ll << 40), AVEY_ERR_UNSUPPORTED, "avey_context: problem too large");
  bf16 *ohi = dt == AVEY_BF16 ? static_cast<bf16 *>(out_lowp) : nullptr;
  bf16 *olo = ohi ? ohi + rows * d : nullptr;
  const long long units = rows * (d / 8);
  const int grid = static_cast<int>(std::min<long long>((units + 255) / 256, 16ll * sm_count()));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dt == AVEY_BF16)
    context_rows<true><<<grid, 256, 0, s>>>(x, N, d, S, k, static_cast<int>(n), idx, w, out, ohi,
                                            olo, units, device_status_word());
  else
    context_rows<false><<<grid, 256, 0, s>>>(x, N, d, S, k, static_cast<int>(n), idx, w, out,
                                             nullptr, nullptr, units, device_status_word());
  AVEY_CHECK_LAUNCH("context_rows", s);
  return AVEY_OK;
}
