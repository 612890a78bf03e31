// avey_layer.cu -- one neural-processor layer (papernotes 整体框架, 关键设计 2-3;
// paperlayer summary §3, App. A):
//   Z = relu(xin U + b)^2;  Z_h | Z_t;  c = V Z_t or Gt Z_t;  x' = x + [Z_h||c] O
//
// bf16 path (AVEY_BF16): enricher and fuser are tcgen05 kernels (avey_tc.cu)
// on bf16 split-pair activations; the mix runs in place on the tail columns
// of the Z split pair, so the fuser reads [Z_h || c] as one [T, m] operand.
// fp32 path (AVEY_F32): SIMT GEMMs with the same fused epilogues.
// Optional prenorm: a row kernel computes 1/sqrt(mean(x^2) + 1e-6) and the
// enricher epilogue scales its accumulator row by it (scaling a row of X
// commutes with X U), so the residual stream itself is never rewritten.
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

__global__ void __launch_bounds__(256) row_inv_rms(const float *__restrict__ x, int T, int d,
                                                   float *__restrict__ inv) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  const float *src = x + row * d;
  float ss = 0.f;
  for (int j = lane * 4; j < d; j += 128) {
    const float4 v = *reinterpret_cast<const float4 *>(src + j);
    ss = fmaf(v.x, v.x, ss);
    ss = fmaf(v.y, v.y, ss);
    ss = fmaf(v.z, v.z, ss);
    ss = fmaf(v.w, v.w, ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (lane == 0) inv[row] = 1.0f / sqrtf(ss / static_cast<float>(d) + 1e-6f);
}

// The same scale from the split pair of x.  hi + lo is the value exactly, and
// every lane visits the same four columns in the same order as row_inv_rms,
// so both give bit-identical scales for the same values.
__global__ void __launch_bounds__(256) row_inv_rms_pair(const bf16 *__restrict__ hi,
                                                        const bf16 *__restrict__ lo, int T, int d,
                                                        float *__restrict__ inv) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= T) return;
  float ss = 0.f;
  for (int j = lane * 4; j < d; j += 128) {
    const uint2 h = *reinterpret_cast<const uint2 *>(hi + row * d + j);
    const uint2 l = *reinterpret_cast<const uint2 *>(lo + row * d + j);
    const float2 h0 = unpack_bf16(h.x), h1 = unpack_bf16(h.y);
    const float2 l0 = unpack_bf16(l.x), l1 = unpack_bf16(l.y);
    const float v0 = h0.x + l0.x, v1 = h0.y + l0.y, v2 = h1.x + l1.x, v3 = h1.y + l1.y;
    ss = fmaf(v0, v0, ss);
    ss = fmaf(v1, v1, ss);
    ss = fmaf(v2, v2, ss);
    ss = fmaf(v3, v3, ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if (lane == 0) inv[row] = 1.0f / sqrtf(ss / static_cast<float>(d) + 1e-6f);
}

__global__ void __launch_bounds__(256) split_rows(const float *__restrict__ x, long long count,
                                                  bf16 *__restrict__ hi, bf16 *__restrict__ lo) {
  const long long i = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) * 8;
  if (i >= count) return;
  const float4 a = *reinterpret_cast<const float4 *>(x + i);
  const float4 b = *reinterpret_cast<const float4 *>(x + i + 4);
  uint32_t h[4], l[4];
  split_pack(a.x, a.y, h[0], l[0]);
  split_pack(a.z, a.w, h[1], l[1]);
  split_pack(b.x, b.y, h[2], l[2]);
  split_pack(b.z, b.w, h[3], l[3]);
  *reinterpret_cast<uint4 *>(hi + i) = make_uint4(h[0], h[1], h[2], h[3]);
  *reinterpret_cast<uint4 *>(lo + i) = make_uint4(l[0], l[1], l[2], l[3]);
}

// fp32 SIMT GEMM C[M, N] = A[M, K] B[N, K]^T with a fused epilogue:
//   ENRICH: C = relu(scale_row * acc + bias)^2 -> out (ld = N)
//   FUSE:   C = resid + acc                    -> out (ld = N)
enum { F32_ENRICH = 0, F32_FUSE = 1 };

template <int MODE>
__global__ void __launch_bounds__(256) gemm_f32(const float *__restrict__ A, const float *__restrict__ Bw,
                                                int M, int N, int K, const float *__restrict__ bias,
                                                const float *__restrict__ inv_rms,
                                                const float *resid, float *out) {
  __shared__ float As[16][64 + 1];
  __shared__ float Bs[16][64 + 1];
  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;  // 16 x 16 threads, 4 x 4 outputs each
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = tid; e < 64 * 16; e += 256) {
      const int r = e / 16, kk = e % 16;
      As[kk][r] = (m0 + r < M && k0 + kk < K) ? A[static_cast<long long>(m0 + r) * K + k0 + kk] : 0.f;
      Bs[kk][r] = (n0 + r < N && k0 + kk < K) ? Bw[static_cast<long long>(n0 + r) * K + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][tr * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tc * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = m0 + tr * 4 + i;
    if (r >= M) continue;
    const float sc = (MODE == F32_ENRICH && inv_rms) ? inv_rms[r] : 1.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c = n0 + tc * 4 + j;
      if (c >= N) continue;
      const long long o = static_cast<long long>(r) * N + c;
      if (MODE == F32_ENRICH) {
        const float v = fmaxf(fmaf(acc[i][j], sc, bias[c]), 0.f);
        out[o] = v * v;
      } else {
        out[o] = resid[o] + acc[i][j];
      }
    }
  }
}

inline size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

}  // namespace
}  // namespace avey

using namespace avey;

extern "C" size_t avey_layer_workspace_bytes(avey_dtype dt, int T, int d, int m, int prenorm) {
  if (T <= 0 || d <= 0 || m <= 0) return 0;
  size_t b = 0;
  if (dt == AVEY_F32) {
    b += align256(static_cast<size_t>(T) * m * 4);  // Z
  } else {
    b += align256(static_cast<size_t>(T) * m * 4);  // Z split pair
    b += align256(static_cast<size_t>(T) * d * 4);  // x_in split pair when none is given
  }
  if (prenorm) b += align256(static_cast<size_t>(T) * 4);
  return b;
}

extern "C" size_t avey_layer_workspace_bytes_ex(avey_dtype dt, int T, int d, int m, int prenorm,
                                                int S, avey_ctx_kind kind) {
  size_t b = avey_layer_workspace_bytes(dt, T, d, m, prenorm);
  if (b && dt == AVEY_BF16 && S > 128 && T % S == 0 && m > 0) {
    b += align256(static_cast<size_t>(T) * m * 4);  // c split pair (T x m_t, m_t < m)
    if (kind == AVEY_DYNAMIC) b += align256(long_dynamic_ws_bytes(T / S, S));
  }
  return b;
}

extern "C" avey_status avey_layer_forward(const avey_layer_params *p, avey_dtype dt, int T,
                                          const float *x_in, const void *x_in_lowp, float *x_out,
                                          void *x_out_lowp, void *ws, size_t ws_bytes,
                                          avey_stream_t stream) {
  return avey_layer_forward_ex(p, dt, T, x_in, x_in_lowp, nullptr, x_out, x_out_lowp, nullptr, ws,
                               ws_bytes, stream);
}

extern "C" avey_status avey_layer_forward_ex(const avey_layer_params *p, avey_dtype dt, int T,
                                             const float *x_in, const void *x_in_lowp,
                                             const float *x_in_rms, float *x_out,
                                             void *x_out_lowp, float *x_out_rms, void *ws,
                                             size_t ws_bytes, avey_stream_t stream) {
  AVEY_REQUIRE(p != nullptr, AVEY_ERR_INVALID_ARG, "avey_layer_forward: null params");
  AVEY_REQUIRE(dt == AVEY_F32 || dt == AVEY_BF16, AVEY_ERR_UNSUPPORTED,
               "avey_layer_forward: dtype %d unsupported (F32 or BF16)", int(dt));
  const int d = p->d, m = p->m, m_h = p->m_h, S = p->S;
  const int mt = m - m_h;
  AVEY_REQUIRE(ws && p->Ut && p->bU && p->Ot, AVEY_ERR_INVALID_ARG,
               "avey_layer_forward: null pointer");
  AVEY_REQUIRE(x_in || (dt == AVEY_BF16 && x_in_lowp), AVEY_ERR_INVALID_ARG,
               "avey_layer_forward: x_in may be NULL only for AVEY_BF16 with x_in_lowp");
  AVEY_REQUIRE(x_out || (dt == AVEY_BF16 && x_out_lowp), AVEY_ERR_INVALID_ARG,
               "avey_layer_forward: x_out may be NULL only for AVEY_BF16 with x_out_lowp");
  AVEY_REQUIRE(p->kind == AVEY_STATIC || p->kind == AVEY_DYNAMIC ||
                   p->kind == AVEY_COUPLED_CAUSAL,
               AVEY_ERR_INVALID_ARG, "avey_layer_forward: bad kind %d", int(p->kind));
  AVEY_REQUIRE(p->kind == AVEY_DYNAMIC || p->V != nullptr, AVEY_ERR_INVALID_ARG,
               "avey_layer_forward: static and coupled layers need V");
  AVEY_REQUIRE(T >= 1 && S >= 1 && T % S == 0, AVEY_ERR_INVALID_ARG,
               "avey_layer_forward: T=%d must be a positive multiple of S=%d", T, S);
  AVEY_REQUIRE(d >= 8 && d % 8 == 0 && m % 8 == 0 && m_h % 8 == 0 && m_h > 0 && m_h < m,
               AVEY_ERR_INVALID_ARG, "avey_layer_forward: need d, m, m_h multiples of 8, 0 < m_h < m");
  AVEY_REQUIRE(p->eps >= 0.f, AVEY_ERR_INVALID_ARG, "avey_layer_forward: eps < 0");
  AVEY_REQUIRE((!x_in || aligned16(x_in)) && (!x_out || aligned16(x_out)) && aligned16(p->Ut) &&
                   aligned16(p->Ot) &&
                   aligned16(p->bU) && (!p->V || aligned16(p->V)) &&
                   (!x_in_lowp || aligned16(x_in_lowp)) && (!x_out_lowp || aligned16(x_out_lowp)),
               AVEY_ERR_INVALID_ARG, "avey_layer_forward: pointers must be 16-byte aligned");
  AVEY_REQUIRE((reinterpret_cast<uintptr_t>(ws) & 255) == 0, AVEY_ERR_INVALID_ARG,
               "avey_layer_forward: workspace must be 256-byte aligned");
  AVEY_REQUIRE((!x_in_rms || (reinterpret_cast<uintptr_t>(x_in_rms) & 3) == 0) &&
                   (!x_out_rms || (reinterpret_cast<uintptr_t>(x_out_rms) & 3) == 0),
               AVEY_ERR_INVALID_ARG, "avey_layer_forward: row scales must be 4-byte aligned");
  AVEY_REQUIRE(!x_out_rms || x_out_rms != x_in_rms, AVEY_ERR_INVALID_ARG,
               "avey_layer_forward: x_out_rms must not be x_in_rms");
  const size_t need = avey_layer_workspace_bytes_ex(dt, T, d, m, p->prenorm, S, p->kind);
  AVEY_REQUIRE(ws_bytes >= need, AVEY_ERR_INVALID_ARG,
               "avey_layer_forward: workspace %zu bytes < %zu required", ws_bytes, need);
  if (dt == AVEY_BF16) {
    AVEY_REQUIRE(S == 16 || S == 32 || S == 64 || S == 128 ||
                     ((S == 256 || S == 512) && p->kind != AVEY_COUPLED_CAUSAL),
                 AVEY_ERR_UNSUPPORTED,
                 "avey_layer_forward(BF16): S=%d unsupported (16, 32, 64 or 128; 256 or 512 for "
                 "static and dynamic layers)", S);
    AVEY_REQUIRE(S <= 128 || m_h % 64 == 0, AVEY_ERR_UNSUPPORTED,
                 "avey_layer_forward(BF16): blocks of %d tokens need m_h %% 64 == 0 (m_h = %d)", S, m_h);
    AVEY_REQUIRE(S <= 128 || p->kind != AVEY_DYNAMIC || m - m_h <= 1024, AVEY_ERR_UNSUPPORTED,
                 "avey_layer_forward(BF16): dynamic blocks of %d tokens need m - m_h <= 1024", S);
  } else {
    AVEY_REQUIRE(S <= 64 && (S & (S - 1)) == 0, AVEY_ERR_UNSUPPORTED,
                 "avey_layer_forward(F32): S=%d unsupported (power of two <= 64)", S);
  }

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char *w = static_cast<char *>(ws);
  const int blocks = T / S;
  avey_status st;

  if (dt == AVEY_F32) {
    float *Z = reinterpret_cast<float *>(w);
    const float *inv = nullptr;
    if (p->prenorm && x_in_rms) {
      inv = x_in_rms;  // the scales of x_in, as a previous layer wrote them
    } else if (p->prenorm) {
      float *iw = reinterpret_cast<float *>(w + align256(static_cast<size_t>(T) * m * 4));
      row_inv_rms<<<(T + 7) / 8, 256, 0, s>>>(x_in, T, d, iw);
      AVEY_CHECK_LAUNCH("row_inv_rms", s);
      inv = iw;
    }
    gemm_f32<F32_ENRICH><<<dim3((m + 63) / 64, (T + 63) / 64), 256, 0, s>>>(
        x_in, static_cast<const float *>(p->Ut), T, m, d, p->bU, inv, nullptr, Z);
    AVEY_CHECK_LAUNCH("gemm_f32_enrich", s);
    if (p->kind == AVEY_STATIC)
      st = launch_static_mix_f32(static_cast<const float *>(p->V), Z + m_h, m, Z + m_h, m, blocks, S,
                                 mt, s);
    else if (p->kind == AVEY_DYNAMIC)
      st = launch_dynamic_mix_f32(Z + m_h, m, Z + m_h, m, blocks, S, mt, p->eps, s);
    else
      st = launch_coupled_mix_f32(static_cast<const float *>(p->V), Z + m_h, m, Z + m_h, m, blocks,
                                  S, mt, s);
    if (st != AVEY_OK) return st;
    gemm_f32<F32_FUSE><<<dim3((d + 63) / 64, (T + 63) / 64), 256, 0, s>>>(
        Z, static_cast<const float *>(p->Ot), T, d, m, nullptr, nullptr, x_in, x_out);
    AVEY_CHECK_LAUNCH("gemm_f32_fuse", s);
    if (x_out_rms) {
      row_inv_rms<<<(T + 7) / 8, 256, 0, s>>>(x_out, T, d, x_out_rms);
      AVEY_CHECK_LAUNCH("row_inv_rms", s);
    }
    return AVEY_OK;
  }

  // bf16 tensor-core path
  const size_t zbytes = align256(static_cast<size_t>(T) * m * 4);
  const size_t xbytes = align256(static_cast<size_t>(T) * d * 4);
  bf16 *Zhi = reinterpret_cast<bf16 *>(w);
  bf16 *Zlo = Zhi + static_cast<long long>(T) * m;
  const bf16 *xhi, *xlo;
  if (x_in_lowp) {
    xhi = static_cast<const bf16 *>(x_in_lowp);
    xlo = xhi + static_cast<long long>(T) * d;
  } else {
    bf16 *h = reinterpret_cast<bf16 *>(w + zbytes);
    bf16 *l = h + static_cast<long long>(T) * d;
    const long long cnt = static_cast<long long>(T) * d;
    split_rows<<<static_cast<unsigned>((cnt / 8 + 255) / 256), 256, 0, s>>>(x_in, cnt, h, l);
    AVEY_CHECK_LAUNCH("split_rows", s);
    xhi = h;
    xlo = l;
  }
  const float *inv = nullptr;
  if (p->prenorm && x_in_rms) {
    inv = x_in_rms;  // the scales of x_in, as a previous layer's fuser wrote them
  } else if (p->prenorm) {
    float *iw = reinterpret_cast<float *>(w + zbytes + xbytes);
    if (x_in)
      row_inv_rms<<<(T + 7) / 8, 256, 0, s>>>(x_in, T, d, iw);
    else
      row_inv_rms_pair<<<(T + 7) / 8, 256, 0, s>>>(xhi, xlo, T, d, iw);
    AVEY_CHECK_LAUNCH("row_inv_rms", s);
    inv = iw;
  }
  st = launch_enrich_tc(xhi, xlo, T, d, static_cast<const bf16 *>(p->Ut), m, p->bU, inv, Zhi, Zlo, s);
  if (st != AVEY_OK) return st;
  const int64_t plane = static_cast<int64_t>(T) * m;
  if (S > 128) {
    // blocks of (k+1)S tokens (the processor without compression): c goes to
    // its own split pair, and the fuser reads [Z_h || c] from the two buffers
    const size_t base = avey_layer_workspace_bytes(dt, T, d, m, p->prenorm);
    bf16 *Chi = reinterpret_cast<bf16 *>(w + base);
    bf16 *Clo = Chi + static_cast<long long>(T) * mt;
    if (p->kind == AVEY_STATIC) {
      st = launch_long_mix_tc(static_cast<const bf16 *>(p->V), nullptr, false, Zhi + m_h, Zlo + m_h,
                              m, blocks, S, mt, Chi, Clo, s);
    } else {
      void *gws = w + base + align256(static_cast<size_t>(T) * m * 4);
      st = launch_long_dynamic_gt(Zhi + m_h, m, blocks, S, mt, p->eps, gws, s);
      if (st != AVEY_OK) return st;
      const bf16 *gt = static_cast<const bf16 *>(gws);
      st = launch_long_mix_tc(gt, gt + static_cast<long long>(blocks) * S * S, true, Zhi + m_h,
                              Zlo + m_h, m, blocks, S, mt, Chi, Clo, s);
    }
    if (st != AVEY_OK) return st;
    bf16 *ohi = static_cast<bf16 *>(x_out_lowp);
    bf16 *olo = ohi ? ohi + static_cast<long long>(T) * d : nullptr;
    return launch_fuse_tc(Zhi, Zlo, T, m, static_cast<const bf16 *>(p->Ot), d, x_in, xhi, xlo, x_out,
                          ohi, olo, s, Chi, Clo, m_h, x_out_rms);
  } else if (p->kind == AVEY_STATIC)
    st = launch_static_mix_x2(static_cast<const bf16 *>(p->V), Zhi + m_h, m, blocks, S, mt, plane,
                              Zhi + m_h, m, plane, s);
  else if (p->kind == AVEY_DYNAMIC)
    st = launch_dynamic_mix_x2(Zhi + m_h, m, plane, Zhi + m_h, m, plane, blocks, S, mt, p->eps, s);
  else
    st = launch_coupled_mix_x2(static_cast<const bf16 *>(p->V), Zhi + m_h, m, plane, Zhi + m_h, m,
                               plane, blocks, S, mt, s);
  if (st != AVEY_OK) return st;
  bf16 *ohi = static_cast<bf16 *>(x_out_lowp);
  bf16 *olo = ohi ? ohi + static_cast<long long>(T) * d : nullptr;
  return launch_fuse_tc(Zhi, Zlo, T, m, static_cast<const bf16 *>(p->Ot), d, x_in, xhi, xlo, x_out, ohi,
                        olo, s, nullptr, nullptr, 0, x_out_rms);
}
