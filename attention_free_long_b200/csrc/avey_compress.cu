// avey_compress.cu -- neural compression of each split with its retrieved
// splits, plus the residual to the split's own tokens (papernotes 关键设计 4,
// eq. 8; paperlayer summary §4.3, App. H):
//   out(t) = sum_{r=0..k} w_r P_r X_{c_r} + X_t,   c_0 = t, w_0 = 1,
// where P_r = P[:, rS:(r+1)S] is the r-th S x S block of P.  Writing the
// product block by block is the same contraction as P X_cat with the weighted
// blocks stacked in rank order; the weight multiplies the fp32 partial
// product of its block, so the bf16 embeddings are never re-rounded.
//
// bf16 kernel (S = 16 and 32; S = 64 and 128 run on tcgen05 in
// avey_compress_tc.cu): one CTA per (target split, column slab of d).  Each retrieved
// block (S rows x slab) and its P_r are staged in shared memory with
// cp.async, double-buffered over r; 8 warps compute the S x slab product with
// mma.sync m16n8k16 (P_r from ldmatrix, X from ldmatrix.trans).  The kernel is
// bound by HBM: it reads (k+1) S x d bf16 per split and writes S x d fp32 plus
// the bf16 split pair.
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

template <int S>
struct CompressTile {
  static constexpr int WM = S >= 32 ? 32 : 16;         // rows per warp
  static constexpr int WARPS_M = S / WM;
  static constexpr int WARPS_N = 8 / WARPS_M;
  static constexpr int WN = 32;                         // columns per warp
  static constexpr int NS = WN * WARPS_N;               // slab width
  static constexpr int MI = WM / 16, NI = WN / 8;
  static constexpr int XLD = NS + 8;                    // padded smem row (elements)
  static constexpr int PLD = S + 8;
  static constexpr int XBYTES = S * XLD * 2;
  static constexpr int PBYTES = S * PLD * 2;
  static constexpr int STAGE = XBYTES + PBYTES;
  static constexpr int NST = S >= 128 ? 2 : (S == 32 ? 3 : 4);  // cp.async depth over the k+1 blocks (2 CTAs / SM at S = 64)
  // output staging (reuses the pipeline buffers): fp32 [S][NS+4], hi/lo [S][NS+8]
  static constexpr int OLD32 = NS + 4;
  static constexpr int OUT_BYTES = S * OLD32 * 4 + 2 * S * XLD * 2;
  static constexpr int SMEM = NST * STAGE > OUT_BYTES ? NST * STAGE : OUT_BYTES;
};

template <int S>
__global__ void __launch_bounds__(256) compress_bf16(const bf16 *__restrict__ x, int N, int d,
                                                     int n, int k, const int32_t *__restrict__ idx,
                                                     const float *__restrict__ w,
                                                     const bf16 *__restrict__ P,
                                                     float *__restrict__ out,
                                                     bf16 *__restrict__ out_hi,
                                                     bf16 *__restrict__ out_lo, long long plane,
                                                     int t0, int nr, int *status) {
  using C = CompressTile<S>;
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ int s_c[33];
  __shared__ float s_w[33];
  // target split t = t0 + blockIdx.y; its idx / w row and its output rows
  // are the blockIdx.y-th of the nr targets handled by this launch
  const int slab = blockIdx.x, tl = blockIdx.y, t = t0 + tl, b = blockIdx.z;
  const int q0 = slab * C::NS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int wm = warp / C::WARPS_N, wn = warp % C::WARPS_N;
  if (tid <= k) {
    int c = t;
    float wr = 1.f;
    if (tid > 0) {
      const long long o = (static_cast<long long>(b) * nr + tl) * k + (tid - 1);
      c = idx[o];
      wr = w[o];
      if (c < -1 || c >= n) {
        record_status(status, AVEY_ERR_DEVICE_BOUNDS);
        c = -1;
      }
    }
    s_c[tid] = c;
    s_w[tid] = wr;
  }
  __syncthreads();

  // Stage r: X block of split s_c[r] (rows, slab columns) and P_r.
  auto load_stage = [&](int r, int buf) {
    uint8_t *xs = smem + buf * C::STAGE;
    uint8_t *ps = xs + C::XBYTES;
    const int c = s_c[r];
    constexpr int XCH = S * (C::NS / 8);  // 16-byte chunks
    for (int e = tid; e < XCH; e += 256) {
      const int row = e / (C::NS / 8), cc = e % (C::NS / 8);
      const int tok = c * S + row, col = q0 + cc * 8;
      const bool ok = c >= 0 && tok < N && col < d;
      const bf16 *src = ok ? x + (static_cast<long long>(b) * N + tok) * d + col : x;
      cp_async16(smem_u32(xs + (row * C::XLD + cc * 8) * 2), src, ok ? 16 : 0);
    }
    constexpr int PCH = S * (S / 8);
    for (int e = tid; e < PCH; e += 256) {
      const int row = e / (S / 8), cc = e % (S / 8);
      const bf16 *src = P + static_cast<long long>(row) * (k + 1) * S + r * S + cc * 8;
      cp_async16(smem_u32(ps + (row * C::PLD + cc * 8) * 2), src, 16);
    }
    cp_async_commit();
  };

  float acc[C::MI][C::NI][4];
#pragma unroll
  for (int i = 0; i < C::MI; ++i)
#pragma unroll
    for (int j = 0; j < C::NI; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[i][j][q] = 0.f;

  // Prologue: blocks 0 .. NST-2 in flight; every iteration then commits one
  // group (possibly empty) so that "all but NST-1 groups done" means block r.
#pragma unroll
  for (int r = 0; r < C::NST - 1; ++r) {
    if (r <= k) load_stage(r, r);
    else cp_async_commit();
  }
  for (int r = 0; r <= k; ++r) {
    if (r + C::NST - 1 <= k) load_stage(r + C::NST - 1, (r + C::NST - 1) % C::NST);
    else cp_async_commit();
    cp_async_wait<C::NST - 1>();
    __syncthreads();
    const uint8_t *xs = smem + (r % C::NST) * C::STAGE;
    const uint8_t *ps = xs + C::XBYTES;
    const float wr = s_w[r];
    // The fp32 partial product of this block (tmp) is scaled by its weight
    // and added to acc; each P_r fragment is loaded once per k step.
    float tmp[C::MI][C::NI][4];
#pragma unroll
    for (int i = 0; i < C::MI; ++i)
#pragma unroll
      for (int j = 0; j < C::NI; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) tmp[i][j][q] = 0.f;
#pragma unroll
    for (int kk = 0; kk < S; kk += 16) {
      uint32_t af[C::MI][4];
#pragma unroll
      for (int i = 0; i < C::MI; ++i) {
        const int row = wm * C::WM + i * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int col = kk + (lane >> 4) * 8;
        ldsm_x4(smem_u32(ps + (row * C::PLD + col) * 2), af[i][0], af[i][1], af[i][2], af[i][3]);
      }
#pragma unroll
      for (int j = 0; j < C::NI; j += 2) {
        uint32_t b0, b1, b2, b3;
        const int krow = kk + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ncol = wn * C::WN + j * 8 + (lane >> 4) * 8;
        ldsm_x4_t(smem_u32(xs + (krow * C::XLD + ncol) * 2), b0, b1, b2, b3);
        const uint32_t bA[2] = {b0, b1}, bB[2] = {b2, b3};
#pragma unroll
        for (int i = 0; i < C::MI; ++i) {
          mma16816(tmp[i][j], af[i], bA);
          mma16816(tmp[i][j + 1], af[i], bB);
        }
      }
    }
#pragma unroll
    for (int i = 0; i < C::MI; ++i)
#pragma unroll
      for (int j = 0; j < C::NI; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[i][j][q] = fmaf(wr, tmp[i][j][q], acc[i][j][q]);
    if (r == 0) {
      // residual: the target split's own tokens (stage 0 holds X_t)
#pragma unroll
      for (int i = 0; i < C::MI; ++i)
#pragma unroll
        for (int j = 0; j < C::NI; ++j)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int row = wm * C::WM + i * 16 + (lane >> 2) + h * 8;
            const int col = wn * C::WN + j * 8 + (lane & 3) * 2;
            const float2 xv = unpack_bf16(*reinterpret_cast<const uint32_t *>(xs + (row * C::XLD + col) * 2));
            acc[i][j][2 * h] += xv.x;
            acc[i][j][2 * h + 1] += xv.y;
          }
    }
    __syncthreads();
  }

  // Stage the fp32 result and its split pair in shared memory (the pipeline
  // buffers are free after the last block), then write them with coalesced
  // 16-byte stores.
  float *o32 = reinterpret_cast<float *>(smem);
  uint8_t *ohi = smem + S * C::OLD32 * 4;
  uint8_t *olo = ohi + S * C::XLD * 2;
  const bool pair = out_hi != nullptr;
#pragma unroll
  for (int i = 0; i < C::MI; ++i)
#pragma unroll
    for (int j = 0; j < C::NI; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = wm * C::WM + i * 16 + (lane >> 2) + h * 8;
        const int col = wn * C::WN + j * 8 + (lane & 3) * 2;
        const float v0 = acc[i][j][2 * h], v1 = acc[i][j][2 * h + 1];
        *reinterpret_cast<float2 *>(o32 + row * C::OLD32 + col) = make_float2(v0, v1);
        if (pair) {
          uint32_t hi, lo;
          split_pack(v0, v1, hi, lo);
          *reinterpret_cast<uint32_t *>(ohi + (row * C::XLD + col) * 2) = hi;
          *reinterpret_cast<uint32_t *>(olo + (row * C::XLD + col) * 2) = lo;
        }
      }
  __syncthreads();
  const long long row0 = (static_cast<long long>(b) * nr + tl) * S;
  for (int e = tid; out != nullptr && e < S * (C::NS / 4); e += 256) {
    const int row = e / (C::NS / 4), cc = e % (C::NS / 4);
    const int col = q0 + cc * 4;
    if (col >= d) continue;
    *reinterpret_cast<float4 *>(out + (row0 + row) * d + col) =
        *reinterpret_cast<const float4 *>(o32 + row * C::OLD32 + cc * 4);
  }
  if (pair) {
    for (int e = tid; e < S * (C::NS / 8); e += 256) {
      const int row = e / (C::NS / 8), cc = e % (C::NS / 8);
      const int col = q0 + cc * 8;
      if (col >= d) continue;
      const long long o = (row0 + row) * d + col;
      *reinterpret_cast<uint4 *>(out_hi + o) = *reinterpret_cast<const uint4 *>(ohi + (row * C::XLD + cc * 8) * 2);
      *reinterpret_cast<uint4 *>(out_lo + o) = *reinterpret_cast<const uint4 *>(olo + (row * C::XLD + cc * 8) * 2);
    }
  }
  (void)plane;
}

// fp32 SIMT compression: one CTA per (target split, 64-column slab).
template <int S>
__global__ void __launch_bounds__(256) compress_f32(const float *__restrict__ x, int N, int d,
                                                    int n, int k, const int32_t *__restrict__ idx,
                                                    const float *__restrict__ w,
                                                    const float *__restrict__ P,
                                                    float *__restrict__ out, int t0, int nr,
                                                    int *status) {
  constexpr int NSL = 64;
  constexpr int PER = (S * NSL + 255) / 256;  // outputs per thread
  __shared__ float xs[S][NSL];
  __shared__ float ps[S][S];
  __shared__ int s_c[33];
  __shared__ float s_w[33];
  const int slab = blockIdx.x, tl = blockIdx.y, t = t0 + tl, b = blockIdx.z, tid = threadIdx.x;
  const int q0 = slab * NSL;
  if (tid <= k) {
    int c = t;
    float wr = 1.f;
    if (tid > 0) {
      const long long o = (static_cast<long long>(b) * nr + tl) * k + (tid - 1);
      c = idx[o];
      wr = w[o];
      if (c < -1 || c >= n) {
        record_status(status, AVEY_ERR_DEVICE_BOUNDS);
        c = -1;
      }
    }
    s_c[tid] = c;
    s_w[tid] = wr;
  }
  __syncthreads();
  float acc[PER], res[PER];
#pragma unroll
  for (int p = 0; p < PER; ++p) acc[p] = res[p] = 0.f;
  for (int r = 0; r <= k; ++r) {
    const int c = s_c[r];
    for (int e = tid; e < S * NSL; e += 256) {
      const int row = e / NSL, col = e % NSL;
      const int tok = c * S + row;
      xs[row][col] = (c >= 0 && tok < N && q0 + col < d)
                         ? x[(static_cast<long long>(b) * N + tok) * d + q0 + col]
                         : 0.f;
    }
    for (int e = tid; e < S * S; e += 256) {
      const int row = e / S, j = e % S;
      ps[row][j] = P[static_cast<long long>(row) * (k + 1) * S + r * S + j];
    }
    __syncthreads();
    const float wr = s_w[r];
#pragma unroll
    for (int p = 0; p < PER; ++p) {
      const int e = tid + p * 256;
      if (e < S * NSL) {
        const int i = e / NSL, col = e % NSL;
        float s = 0.f;
        for (int j = 0; j < S; ++j) s = fmaf(ps[i][j], xs[j][col], s);
        acc[p] = fmaf(wr, s, acc[p]);
        if (r == 0) res[p] = xs[i][col];
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < PER; ++p) {
    const int e = tid + p * 256;
    if (e < S * NSL) {
      const int i = e / NSL, col = e % NSL;
      if (q0 + col < d)
        out[((static_cast<long long>(b) * nr + tl) * S + i) * d + q0 + col] =
            acc[p] + res[p];
    }
  }
}

template <int S>
avey_status run_compress_bf16(const bf16 *x, int B, int N, int d, int n, int k, int t0, int nr,
                              const int32_t *idx, const float *w, const bf16 *P, float *out,
                              bf16 *hi, bf16 *lo, cudaStream_t s) {
  using C = CompressTile<S>;
  auto kern = compress_bf16<S>;
  if (C::SMEM > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) {
      set_detail("compress: %s", cudaGetErrorString(e));
      return AVEY_ERR_CUDA;
    }
  }
  const dim3 grid((d + C::NS - 1) / C::NS, nr, B);
  const long long plane = static_cast<long long>(B) * nr * S * d;
  kern<<<grid, 256, C::SMEM, s>>>(x, N, d, n, k, idx, w, P, out, hi, lo, plane, t0, nr,
                                  device_status_word());
  AVEY_CHECK_LAUNCH("compress_bf16", s);
  return AVEY_OK;
}

}  // namespace
}  // namespace avey

using namespace avey;

static avey_status compress_range(const void *x, avey_dtype dt, int B, int N, int d, int S, int k,
                                  int t0, int t1, const int32_t *idx, const float *w,
                                  const void *P, float *out, void *out_lowp, cudaStream_t s,
                                  const char *fn) {
  AVEY_REQUIRE(dt == AVEY_F32 || dt == AVEY_BF16, AVEY_ERR_UNSUPPORTED,
               "%s: dtype %d unsupported (F32 or BF16)", fn, int(dt));
  AVEY_REQUIRE(x && idx && w && P, AVEY_ERR_INVALID_ARG, "%s: null pointer", fn);
  AVEY_REQUIRE(out || (dt == AVEY_BF16 && out_lowp), AVEY_ERR_INVALID_ARG,
               "%s: out may be NULL only for AVEY_BF16 with out_lowp", fn);
  AVEY_REQUIRE(B >= 1 && N >= 1 && d >= 1 && S >= 1 && k >= 1, AVEY_ERR_INVALID_ARG,
               "%s: sizes must be >= 1", fn);
  AVEY_REQUIRE(d % 8 == 0, AVEY_ERR_INVALID_ARG, "%s: d=%d must be a multiple of 8", fn, d);
  AVEY_REQUIRE(k <= 32, AVEY_ERR_UNSUPPORTED, "%s: k=%d > 32", fn, k);
  AVEY_REQUIRE(aligned16(x) && aligned16(P) && (!out || aligned16(out)) && (!out_lowp || aligned16(out_lowp)),
               AVEY_ERR_INVALID_ARG, "%s: pointers must be 16-byte aligned", fn);
  const int n = (N + S - 1) / S;
  AVEY_REQUIRE(0 <= t0 && t0 <= t1 && t1 <= n && t1 - t0 <= 65535, AVEY_ERR_INVALID_ARG,
               "%s: target range [%d, %d) outside [0, %d) or wider than 65535", fn, t0, t1, n);
  const int nr = t1 - t0;
  if (nr == 0) return AVEY_OK;
  if (dt == AVEY_BF16) {
    AVEY_REQUIRE(S == 16 || S == 32 || S == 64 || S == 128, AVEY_ERR_UNSUPPORTED,
                 "%s(BF16): S=%d unsupported (16, 32, 64 or 128)", fn, S);
    const bf16 *xb = static_cast<const bf16 *>(x);
    const bf16 *Pb = static_cast<const bf16 *>(P);
    bf16 *hi = static_cast<bf16 *>(out_lowp);
    bf16 *lo = hi ? hi + static_cast<long long>(B) * nr * S * d : nullptr;
    // S = 64 and 128 run on tcgen05 (d % 8 == 0 is checked above), the
    // smaller splits on the mma.sync kernel
    if (compress_tc_supported(S, d))
      return launch_compress_tc(xb, B, N, d, S, k, t0, nr, idx, w, Pb, out, hi, lo, s);
    if (S == 16) return run_compress_bf16<16>(xb, B, N, d, n, k, t0, nr, idx, w, Pb, out, hi, lo, s);
    return run_compress_bf16<32>(xb, B, N, d, n, k, t0, nr, idx, w, Pb, out, hi, lo, s);
  }
  AVEY_REQUIRE(S <= 64 && (S & (S - 1)) == 0, AVEY_ERR_UNSUPPORTED,
               "%s(F32): S=%d unsupported (power of two <= 64)", fn, S);
  const dim3 grid((d + 63) / 64, nr, B);
  const float *xf = static_cast<const float *>(x);
  const float *Pf = static_cast<const float *>(P);
  int *st = device_status_word();
  switch (S) {
#define AVEY_CF_CASE(SS) \
  case SS: compress_f32<SS><<<grid, 256, 0, s>>>(xf, N, d, n, k, idx, w, Pf, out, t0, nr, st); break;
    AVEY_CF_CASE(1) AVEY_CF_CASE(2) AVEY_CF_CASE(4) AVEY_CF_CASE(8) AVEY_CF_CASE(16)
    AVEY_CF_CASE(32) AVEY_CF_CASE(64)
#undef AVEY_CF_CASE
  }
  AVEY_CHECK_LAUNCH("compress_f32", s);
  return AVEY_OK;
}

extern "C" avey_status avey_compress(const void *x, avey_dtype dt, int B, int N, int d, int S,
                                     int k, const int32_t *idx, const float *w, const void *P,
                                     float *out, void *out_lowp, avey_stream_t stream) {
  const int n = S >= 1 ? (N + S - 1) / S : 0;
  return compress_range(x, dt, B, N, d, S, k, 0, n, idx, w, P, out, out_lowp,
                        reinterpret_cast<cudaStream_t>(stream), "avey_compress");
}

extern "C" avey_status avey_compress_rows(const void *x, avey_dtype dt, int B, int N, int d, int S,
                                          int k, int t0, int t1, const int32_t *idx,
                                          const float *w, const void *P, float *out,
                                          void *out_lowp, avey_stream_t stream) {
  return compress_range(x, dt, B, N, d, S, k, t0, t1, idx, w, P, out, out_lowp,
                        reinterpret_cast<cudaStream_t>(stream), "avey_compress_rows");
}
