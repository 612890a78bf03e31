// avey_rank.cu -- the Avey-B ranker: row normalisation, MaxSim split scores,
// top-k selection with divide-by-max weights (Avey-B paperlayer summary §3
// Background and App. H; papernotes 整体框架).
//
//   inv_norms        (bf16) 1/max(||x||, 1e-12) per token, 0 for the pad rows
//                    of the last split; the tcgen05 MaxSim (avey_maxsim2.cu,
//                    and avey_tc.cu for S = 16) reads the raw bf16 rows and
//                    applies these scales in its epilogue.
//   normalize_rows   (fp32) N(x) = x / max(||x||, 1e-12) per token, padded to
//                    n*S rows per sequence (pad rows zero).
//   maxsim_f32       SIMT fp32 version (one CTA per target/candidate pair).
//   topk_warp        one warp per target split, one pass over its score row
//                    keeping a warp-wide sorted list of the k best, order
//                    (score desc, index asc), self excluded, behind a bar
//                    seeded from the first batch, then w_r = s_r / s_1 with
//                    IEEE division (s_1 / s_1 == 1).
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

template <typename Tin, typename Tout>
__global__ void __launch_bounds__(256) normalize_rows(const Tin *__restrict__ x, int B, int N,
                                                      int d, int R, Tout *__restrict__ xhat) {
  const long long row = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<long long>(B) * R) return;
  const int b = static_cast<int>(row / R);
  const int tok = static_cast<int>(row - static_cast<long long>(b) * R);
  Tout *dst = xhat + row * d;
  if (tok >= N) {  // pad row
    for (int j = lane * 8; j < d; j += 256) {
      if constexpr (sizeof(Tout) == 2) {
        *reinterpret_cast<uint4 *>(dst + j) = make_uint4(0, 0, 0, 0);
      } else {
        *reinterpret_cast<float4 *>(dst + j) = make_float4(0, 0, 0, 0);
        *reinterpret_cast<float4 *>(dst + j + 4) = make_float4(0, 0, 0, 0);
      }
    }
    return;
  }
  const Tin *src = x + (static_cast<long long>(b) * N + tok) * d;
  float v[8];
  auto load8 = [&](int j) {
    if constexpr (sizeof(Tin) == 2) {
      const uint4 u = *reinterpret_cast<const uint4 *>(src + j);
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = unpack_bf16(w4[q]);
        v[2 * q] = f.x;
        v[2 * q + 1] = f.y;
      }
    } else {
      const float4 a = *reinterpret_cast<const float4 *>(src + j);
      const float4 c = *reinterpret_cast<const float4 *>(src + j + 4);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
      v[4] = c.x; v[5] = c.y; v[6] = c.z; v[7] = c.w;
    }
  };
  float ss = 0.f;
  for (int j = lane * 8; j < d; j += 256) {
    load8(j);
#pragma unroll
    for (int q = 0; q < 8; ++q) ss = fmaf(v[q], v[q], ss);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  const float inv = 1.0f / fmaxf(sqrtf(ss), 1e-12f);
  for (int j = lane * 8; j < d; j += 256) {
    load8(j);
    if constexpr (sizeof(Tout) == 2) {
      *reinterpret_cast<uint4 *>(dst + j) =
          make_uint4(pack_bf16(v[0] * inv, v[1] * inv), pack_bf16(v[2] * inv, v[3] * inv),
                     pack_bf16(v[4] * inv, v[5] * inv), pack_bf16(v[6] * inv, v[7] * inv));
    } else {
      *reinterpret_cast<float4 *>(dst + j) = make_float4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
      *reinterpret_cast<float4 *>(dst + j + 4) =
          make_float4(v[4] * inv, v[5] * inv, v[6] * inv, v[7] * inv);
    }
  }
}

// fp32 MaxSim: one CTA per (target t, candidate c, sequence b).  Thread
// layout: TPR = 256/S threads per target row, each covering S/TPR candidate
// rows; the d-loop is staged through shared memory in chunks of 32.
template <int S>
__global__ void __launch_bounds__(256) maxsim_f32(const float *__restrict__ xhat, int R, int d,
                                                  int n, float *__restrict__ scores) {
  constexpr int TPR = (256 / S) < S ? (256 / S) : S;  // threads per target row
  constexpr int CPT = S / TPR;                         // candidate rows per thread
  __shared__ float st[S][33];
  __shared__ float sc[S][33];
  __shared__ float rowmax[S][TPR];
  const int c = blockIdx.x, t = blockIdx.y, b = blockIdx.z;
  const float *xt = xhat + (static_cast<long long>(b) * R + static_cast<long long>(t) * S) * d;
  const float *xc = xhat + (static_cast<long long>(b) * R + static_cast<long long>(c) * S) * d;
  const int tid = threadIdx.x;
  const int i = tid % S;          // target row
  const int part = tid / S;       // which slice of candidate rows
  const bool active = tid < S * TPR;
  float acc[CPT];
#pragma unroll
  for (int q = 0; q < CPT; ++q) acc[q] = 0.f;
  for (int k0 = 0; k0 < d; k0 += 32) {
    for (int e = tid; e < S * 32; e += 256) {
      const int r = e / 32, kk = e % 32;
      st[r][kk] = (k0 + kk < d) ? xt[static_cast<long long>(r) * d + k0 + kk] : 0.f;
      sc[r][kk] = (k0 + kk < d) ? xc[static_cast<long long>(r) * d + k0 + kk] : 0.f;
    }
    __syncthreads();
    if (active) {
#pragma unroll
      for (int q = 0; q < CPT; ++q) {
        const int j = part * CPT + q;
        float s = acc[q];
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) s = fmaf(st[i][kk], sc[j][kk], s);
        acc[q] = s;
      }
    }
    __syncthreads();
  }
  if (active) {
    float m = acc[0];
#pragma unroll
    for (int q = 1; q < CPT; ++q) m = fmaxf(m, acc[q]);
    rowmax[i][part] = m;
  }
  __syncthreads();
  if (tid == 0) {
    float total = 0.f;
    for (int r = 0; r < S; ++r) {
      float m = rowmax[r][0];
      for (int p = 1; p < TPR; ++p) m = fmaxf(m, rowmax[r][p]);
      total += m;
    }
    scores[(static_cast<long long>(b) * n + t) * n + c] = total;
  }
}

// Rows of inv [B, rs_ld]: rows < N get 1/max(||x||, 1e-12), rows >= N (split
// padding and tile padding) get 0.  A persistent grid of resident blocks; each
// warp takes two rows per step (rows w and w + warps, then on by 2 * warps)
// and issues the 16-byte loads of both rows, four per lane and row for every
// 1024 features, before any use, so that enough bytes are in flight to cover
// HBM latency.  Each lane sums its features in the same order for any grid.
__global__ void __launch_bounds__(256) inv_norms(const bf16 *__restrict__ x, int B, int N, int d,
                                                 int rs_ld, float *__restrict__ inv) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * 8;
  const long long total = static_cast<long long>(B) * rs_ld;
  for (long long r0 = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5); r0 < total;
       r0 += 2 * warps) {
    const bf16 *src[2];
    bool live[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const long long row = r0 + h * warps;
      const int b = static_cast<int>(row / rs_ld);
      const int tok = static_cast<int>(row - static_cast<long long>(b) * rs_ld);
      live[h] = row < total && tok < N;
      src[h] = x + (live[h] ? (static_cast<long long>(b) * N + tok) * d : 0);
    }
    float ss[2] = {0.f, 0.f};
    for (int j0 = lane * 8; j0 < d; j0 += 4 * 256) {
      uint4 u[2][4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int r = 0; r < 4; ++r)
          u[h][r] = live[h] && j0 + r * 256 < d
                        ? *reinterpret_cast<const uint4 *>(src[h] + j0 + r * 256)
                        : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t w4[4] = {u[h][r].x, u[h][r].y, u[h][r].z, u[h][r].w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = unpack_bf16(w4[q]);
            ss[h] = fmaf(f.x, f.x, ss[h]);
            ss[h] = fmaf(f.y, f.y, ss[h]);
          }
        }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float t = ss[h];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
      const long long row = r0 + h * warps;
      if (lane == 0 && row < total) inv[row] = live[h] ? 1.0f / fmaxf(sqrtf(t), 1e-12f) : 0.f;
    }
  }
}

constexpr int kTopkWarps = 8;

// One warp per target split, one pass over its score row.  The warp keeps
// one sorted list of the k best candidates so far, lane q holding the q-th by
// the key (score desc, index asc).  Every loaded element is compared with the
// list's k-th key; the (rare, about k ln(n/k) per row) elements that beat it
// are inserted one at a time, warp-wide: lanes behind the insertion point take
// their predecessor's entry.  Self, and c > t for the unidirectional ranker,
// never enter; -inf and NaN scores never beat the empty list's -inf.  Five
// blocks stay resident per SM (at most 48 registers), which a score matrix
// far past L2 needs to keep HBM busy.
__device__ __forceinline__ bool key_gt(float a, int ia, float b, int ib) {
  return a > b || (a == b && ia < ib);
}

__global__ void __launch_bounds__(kTopkWarps * 32, 5)
    topk_warp(const float *__restrict__ scores, int B, int n, int t0, int nr, int k, int causal,
              int vec4, int32_t *__restrict__ idx, float *__restrict__ w) {
  // rows of this launch: targets t0 .. t0+nr-1 of every sequence; outputs are
  // [B, nr, k]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long rowid = static_cast<long long>(blockIdx.x) * kTopkWarps + warp;
  if (rowid >= static_cast<long long>(B) * nr) return;
  const long long bq = rowid / nr;
  const int t = t0 + static_cast<int>(rowid - bq * nr);
  const float *src = scores + (bq * n + t) * n;
  const int lim = causal ? t : n;  // candidates c < lim, c != t
  float lv = -INFINITY;  // this lane's list entry (q = lane)
  int lc = 0x7fffffff;
  float tv = -INFINITY;  // the bar a new candidate must clear: the list's k-th
  int tc = 0x7fffffff;   // entry, or the seed while the list is not yet full
  float sv = -INFINITY;  // the seed bar (see seed below)
  int sc = 0x7fffffff;
  auto consider = [&](float v, int c) {
    const bool ok = c < lim && c != t && key_gt(v, c, tv, tc);
    unsigned mask = __ballot_sync(0xffffffffu, ok);
    while (mask) {
      const int srcl = __ffs(mask) - 1;
      mask &= mask - 1;
      const float nv = __shfl_sync(0xffffffffu, v, srcl);
      const int nc = __shfl_sync(0xffffffffu, c, srcl);
      if (!key_gt(nv, nc, tv, tc)) continue;  // the bar rose since the ballot
      const int pos = __popc(__ballot_sync(0xffffffffu, lane < k && key_gt(lv, lc, nv, nc)));
      const float pv = __shfl_up_sync(0xffffffffu, lv, 1);
      const int pc = __shfl_up_sync(0xffffffffu, lc, 1);
      if (lane == pos) {
        lv = nv;
        lc = nc;
      } else if (lane > pos) {
        lv = pv;
        lc = pc;
      }
      const float kv = __shfl_sync(0xffffffffu, lv, k - 1);
      const int kc = __shfl_sync(0xffffffffu, lc, k - 1);
      // every entry cleared the seed, so a full list's k-th is at least the seed
      if (key_gt(kv, kc, sv, sc)) {
        tv = kv;
        tc = kc;
      }
    }
  };
  // The seed: every lane offers its best candidate of the first batch, a
  // bitonic network sorts the 32 offers (key order, descending) and the k-th
  // becomes the bar.  k distinct candidates are at least that good, so nothing
  // below it can be chosen; without it the empty list takes nearly every
  // element of the first batch one warp-wide insertion at a time.  The bar is
  // set just below the seed's own key, so the seed itself still enters.
  auto seed = [&](float bv, int bc) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, stride);
        const int oc = __shfl_xor_sync(0xffffffffu, bc, stride);
        const bool desc = (lane & size) == 0 || size == 32;
        const bool keep_greater = desc == ((lane & stride) == 0);
        if (keep_greater == key_gt(ov, oc, bv, bc)) {
          bv = ov;
          bc = oc;
        }
      }
    }
    const float kv = __shfl_sync(0xffffffffu, bv, k - 1);
    const int kc = __shfl_sync(0xffffffffu, bc, k - 1);
    if (kc != 0x7fffffff) {  // k real offers: the k-th is a valid bar
      sv = tv = kv;
      sc = tc = kc + 1;
    }
  };
  auto offer = [&](float v, int c, float &bv, int &bc) {
    if (c < lim && c != t && key_gt(v, c, bv, bc)) {
      bv = v;
      bc = c;
    }
  };
  if (vec4) {
    const float4 *s4 = reinterpret_cast<const float4 *>(src);
    const int n4 = (lim + 3) >> 2;  // float4 groups that hold a candidate
    for (int g0 = 0; g0 < n4; g0 += 128) {
      // four loads in flight per lane, then the warp-uniform screening
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int g = g0 + 32 * u + lane;
        v[u] = g < n4 ? __ldg(s4 + g) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
      }
      if (g0 == 0) {
        float bv = -INFINITY;
        int bc = 0x7fffffff;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = 4 * (32 * u + lane);
          offer(v[u].x, c, bv, bc);
          offer(v[u].y, c + 1, bv, bc);
          offer(v[u].z, c + 2, bv, bc);
          offer(v[u].w, c + 3, bv, bc);
        }
        seed(bv, bc);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        // one warp vote per group of four: the per-element path runs only when
        // some lane's group maximum can clear the bar (its lowest index is the
        // most favourable tie-break)
        const int c = 4 * (g0 + 32 * u + lane);
        const float m = fmaxf(fmaxf(v[u].x, v[u].y), fmaxf(v[u].z, v[u].w));
        if (!__any_sync(0xffffffffu, key_gt(m, c, tv, tc))) continue;
        consider(v[u].x, c);
        consider(v[u].y, c + 1);
        consider(v[u].z, c + 2);
        consider(v[u].w, c + 3);
      }
    }
  } else {
    for (int c0 = 0; c0 < lim; c0 += 128) {
      float v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u + lane;
        v[u] = c < lim ? __ldg(src + c) : -INFINITY;
      }
      if (c0 == 0) {
        float bv = -INFINITY;
        int bc = 0x7fffffff;
#pragma unroll
        for (int u = 0; u < 4; ++u) offer(v[u], 32 * u + lane, bv, bc);
        seed(bv, bc);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) consider(v[u], c0 + 32 * u + lane);
    }
  }
  // lane r < k holds the r-th choice; w_r = s_r / max(s_1, 1e-30)
  const int avail = causal ? t : n - 1;
  const float b0 = __shfl_sync(0xffffffffu, lv, 0);
  const float s1 = b0 > 1e-30f ? b0 : 1e-30f;
  if (lane < k) {
    const long long o = rowid * k + lane;
    const bool valid = lane < avail && lc != 0x7fffffff && lv != -INFINITY;
    idx[o] = valid ? lc : -1;
    w[o] = valid ? lv / s1 : 0.f;
  }
}

inline size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

}  // namespace

avey_status launch_normalize(const void *x, avey_dtype dt, int B, int N, int d, int S, void *xhat,
                             cudaStream_t s) {
  const int n = (N + S - 1) / S, R = n * S;
  const long long rows = static_cast<long long>(B) * R;
  const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
  if (dt == AVEY_BF16)
    normalize_rows<bf16, bf16><<<grid, 256, 0, s>>>(static_cast<const bf16 *>(x), B, N, d, R,
                                                    static_cast<bf16 *>(xhat));
  else
    normalize_rows<float, float><<<grid, 256, 0, s>>>(static_cast<const float *>(x), B, N, d, R,
                                                      static_cast<float *>(xhat));
  AVEY_CHECK_LAUNCH("normalize_rows", s);
  return AVEY_OK;
}

avey_status launch_inv_norms(const bf16 *x, int B, int N, int d, int rs_ld, float *inv,
                             cudaStream_t s) {
  const long long rows = static_cast<long long>(B) * rs_ld;
  const long long blocks = std::min<long long>((rows + 15) / 16, 8ll * sm_count());
  if (blocks <= 0) return AVEY_OK;
  inv_norms<<<static_cast<unsigned>(blocks), 256, 0, s>>>(x, B, N, d, rs_ld, inv);
  AVEY_CHECK_LAUNCH("inv_norms", s);
  return AVEY_OK;
}

avey_status launch_topk_rows(const float *scores, int B, int n, int t0, int nr, int k, int causal,
                             int32_t *idx, float *w, cudaStream_t s) {
  const long long rows = static_cast<long long>(B) * nr;
  if (rows == 0) return AVEY_OK;
  const unsigned grid = static_cast<unsigned>((rows + kTopkWarps - 1) / kTopkWarps);
  const int vec4 = (n % 4 == 0 && aligned16(scores)) ? 1 : 0;
  topk_warp<<<grid, kTopkWarps * 32, 0, s>>>(scores, B, n, t0, nr, k, causal, vec4, idx, w);
  AVEY_CHECK_LAUNCH("topk_warp", s);
  return AVEY_OK;
}

avey_status launch_topk(const float *scores, int B, int n, int k, int causal, int32_t *idx,
                        float *w, cudaStream_t s) {
  return launch_topk_rows(scores, B, n, 0, n, k, causal, idx, w, s);
}

static avey_status launch_maxsim_f32(const float *xhat, int B, int R, int d, int S, int n,
                                     float *scores, cudaStream_t s) {
  const dim3 grid(n, n, B);
  switch (S) {
#define AVEY_MS_CASE(SS)                                                          \
  case SS:                                                                        \
    maxsim_f32<SS><<<grid, 256, 0, s>>>(xhat, R, d, n, scores);                   \
    break;
    AVEY_MS_CASE(1) AVEY_MS_CASE(2) AVEY_MS_CASE(4) AVEY_MS_CASE(8) AVEY_MS_CASE(16)
    AVEY_MS_CASE(32) AVEY_MS_CASE(64) AVEY_MS_CASE(128)
#undef AVEY_MS_CASE
    default:
      set_detail("avey_rank(F32): S=%d unsupported (powers of two up to 128)", S);
      return AVEY_ERR_UNSUPPORTED;
  }
  AVEY_CHECK_LAUNCH("maxsim_f32", s);
  return AVEY_OK;
}

}  // namespace avey

using namespace avey;

// Padded row count of the inverse-norm table: a multiple of the MaxSim
// column tile (256) so that every tile's scale loads stay in bounds.
static inline long long scale_ld(long long R) { return (R + 255) / 256 * 256; }

extern "C" size_t avey_rank_workspace_bytes(avey_dtype dt, int B, int N, int d, int S) {
  if (B <= 0 || N <= 0 || d <= 0 || S <= 0) return 0;
  const long long n = (N + S - 1) / S, R = n * S;
  const size_t first = dt == AVEY_F32 ? static_cast<size_t>(B) * R * d * 4   // normalised copy
                                      : static_cast<size_t>(B) * scale_ld(R) * 4;  // 1/||x||
  return align256(first) + align256(static_cast<size_t>(B) * n * n * 4);
}

extern "C" avey_status avey_rank(const void *x, avey_dtype dt, int B, int N, int d, int S, int k,
                                 int32_t *idx, float *w, float *scores, void *ws, size_t ws_bytes,
                                 avey_stream_t stream) {
  return avey_rank_ex(x, dt, B, N, d, S, k, 0u, idx, w, scores, ws, ws_bytes, stream);
}

extern "C" avey_status avey_topk(const float *scores, int B, int n, int k, uint32_t flags,
                                 int32_t *idx, float *w, avey_stream_t stream) {
  AVEY_REQUIRE(scores && idx && w, AVEY_ERR_INVALID_ARG, "avey_topk: null pointer");
  AVEY_REQUIRE(B >= 1 && n >= 1 && k >= 1, AVEY_ERR_INVALID_ARG,
               "avey_topk: sizes must be >= 1 (B=%d n=%d k=%d)", B, n, k);
  AVEY_REQUIRE(k <= 32, AVEY_ERR_UNSUPPORTED, "avey_topk: k=%d > 32", k);
  AVEY_REQUIRE((flags & ~static_cast<uint32_t>(AVEY_RANK_UNIDIRECTIONAL)) == 0,
               AVEY_ERR_INVALID_ARG, "avey_topk: unknown flags 0x%x", flags);
  AVEY_REQUIRE(static_cast<long long>(B) * n <= (1ll << 31) - 1, AVEY_ERR_UNSUPPORTED,
               "avey_topk: problem too large");
  return launch_topk(scores, B, n, k, (flags & AVEY_RANK_UNIDIRECTIONAL) ? 1 : 0, idx, w,
                     reinterpret_cast<cudaStream_t>(stream));
}

extern "C" avey_status avey_topk_rows(const float *scores, int B, int n, int t0, int t1, int k,
                                      uint32_t flags, int32_t *idx, float *w,
                                      avey_stream_t stream) {
  AVEY_REQUIRE(scores && idx && w, AVEY_ERR_INVALID_ARG, "avey_topk_rows: null pointer");
  AVEY_REQUIRE(B >= 1 && n >= 1 && k >= 1 && k <= 32, AVEY_ERR_INVALID_ARG,
               "avey_topk_rows: sizes (B=%d n=%d, 1 <= k=%d <= 32)", B, n, k);
  AVEY_REQUIRE(0 <= t0 && t0 <= t1 && t1 <= n, AVEY_ERR_INVALID_ARG,
               "avey_topk_rows: target range [%d, %d) outside [0, %d)", t0, t1, n);
  AVEY_REQUIRE((flags & ~static_cast<uint32_t>(AVEY_RANK_UNIDIRECTIONAL)) == 0,
               AVEY_ERR_INVALID_ARG, "avey_topk_rows: unknown flags 0x%x", flags);
  return launch_topk_rows(scores, B, n, t0, t1 - t0, k, (flags & AVEY_RANK_UNIDIRECTIONAL) ? 1 : 0,
                          idx, w, reinterpret_cast<cudaStream_t>(stream));
}

extern "C" avey_status avey_maxsim_part(const void *x, avey_dtype dt, int B, int N, int d, int S,
                                        int part, int nparts, float *scores, void *ws,
                                        size_t ws_bytes, avey_stream_t stream) {
  AVEY_REQUIRE(dt == AVEY_BF16, AVEY_ERR_UNSUPPORTED,
               "avey_maxsim_part: dtype %d unsupported (BF16)", int(dt));
  AVEY_REQUIRE(x && scores && ws, AVEY_ERR_INVALID_ARG, "avey_maxsim_part: null pointer");
  AVEY_REQUIRE(B >= 1 && N >= 1 && d >= 1, AVEY_ERR_INVALID_ARG,
               "avey_maxsim_part: sizes must be >= 1 (B=%d N=%d d=%d)", B, N, d);
  AVEY_REQUIRE(S == 32 || S == 64 || S == 128, AVEY_ERR_UNSUPPORTED,
               "avey_maxsim_part: S=%d unsupported (32, 64 or 128)", S);
  AVEY_REQUIRE(nparts >= 1 && part >= 0 && part < nparts, AVEY_ERR_INVALID_ARG,
               "avey_maxsim_part: part %d of %d", part, nparts);
  AVEY_REQUIRE(d % 8 == 0, AVEY_ERR_INVALID_ARG, "avey_maxsim_part: d=%d must be a multiple of 8", d);
  AVEY_REQUIRE(aligned16(x) && aligned16(scores) && (reinterpret_cast<uintptr_t>(ws) & 255) == 0,
               AVEY_ERR_INVALID_ARG,
               "avey_maxsim_part: x, scores 16-byte and the workspace 256-byte aligned");
  const long long n = (N + S - 1) / S, R = n * S;
  AVEY_REQUIRE(n <= 46340 && static_cast<long long>(B) * R <= (1ll << 31) - 1,
               AVEY_ERR_UNSUPPORTED, "avey_maxsim_part: problem too large");
  const size_t need = avey_rank_workspace_bytes(dt, B, N, d, S);
  AVEY_REQUIRE(ws_bytes >= need, AVEY_ERR_INVALID_ARG,
               "avey_maxsim_part: workspace %zu bytes < %zu required", ws_bytes, need);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  float *inv = static_cast<float *>(ws);
  const int ld = static_cast<int>(scale_ld(R));
  avey_status st = launch_inv_norms(static_cast<const bf16 *>(x), B, N, d, ld, inv, s);
  if (st != AVEY_OK) return st;
  return launch_maxsim_pair(static_cast<const bf16 *>(x), inv, B, N, static_cast<int>(R), ld, d, S,
                            static_cast<int>(n), scores, s, part, nparts);
}

// Shape and dtype checks shared by every ranker entry point (fn names the
// entry point in the error detail).
avey_status avey::check_rank_shape(const char *fn, avey_dtype dt, int B, int N, int d, int S,
                                     int k) {
  AVEY_REQUIRE(dt == AVEY_F32 || dt == AVEY_BF16, AVEY_ERR_UNSUPPORTED,
               "%s: dtype %d unsupported (F32 or BF16)", fn, int(dt));
  AVEY_REQUIRE(B >= 1 && N >= 1 && d >= 1 && S >= 1 && k >= 1, AVEY_ERR_INVALID_ARG,
               "%s: sizes must be >= 1 (B=%d N=%d d=%d S=%d k=%d)", fn, B, N, d, S, k);
  AVEY_REQUIRE(d % 8 == 0, AVEY_ERR_INVALID_ARG, "%s: d=%d must be a multiple of 8", fn, d);
  AVEY_REQUIRE(k <= 32, AVEY_ERR_UNSUPPORTED, "%s: k=%d > 32", fn, k);
  if (dt == AVEY_BF16)
    AVEY_REQUIRE(S == 16 || S == 32 || S == 64 || S == 128, AVEY_ERR_UNSUPPORTED,
                 "%s(BF16): S=%d unsupported (16, 32, 64 or 128)", fn, S);
  else
    AVEY_REQUIRE(S <= 128 && (S & (S - 1)) == 0, AVEY_ERR_UNSUPPORTED,
                 "%s(F32): S=%d unsupported (power of two <= 128)", fn, S);
  const long long n = (N + S - 1) / S, R = n * S;
  AVEY_REQUIRE(n <= 46340 && static_cast<long long>(B) * R <= (1ll << 31) - 1,
               AVEY_ERR_UNSUPPORTED, "%s: problem too large", fn);
  return AVEY_OK;
}

extern "C" avey_status avey_rank_ex(const void *x, avey_dtype dt, int B, int N, int d, int S, int k,
                                    uint32_t flags, int32_t *idx, float *w, float *scores, void *ws,
                                    size_t ws_bytes, avey_stream_t stream) {
  AVEY_REQUIRE((flags & ~static_cast<uint32_t>(AVEY_RANK_UNIDIRECTIONAL)) == 0u,
               AVEY_ERR_INVALID_ARG, "avey_rank: unknown flags 0x%x", flags);
  AVEY_REQUIRE(x && idx && w && ws, AVEY_ERR_INVALID_ARG, "avey_rank: null pointer");
  {
    const avey_status sh = check_rank_shape("avey_rank", dt, B, N, d, S, k);
    if (sh != AVEY_OK) return sh;
  }
  AVEY_REQUIRE(aligned16(x) && aligned16(ws) && (!scores || aligned16(scores)),
               AVEY_ERR_INVALID_ARG, "avey_rank: pointers must be 16-byte aligned");
  AVEY_REQUIRE((reinterpret_cast<uintptr_t>(ws) & 255) == 0, AVEY_ERR_INVALID_ARG,
               "avey_rank: workspace must be 256-byte aligned");
  const long long n = (N + S - 1) / S, R = n * S;
  const size_t need = avey_rank_workspace_bytes(dt, B, N, d, S);
  AVEY_REQUIRE(ws_bytes >= need, AVEY_ERR_INVALID_ARG,
               "avey_rank: workspace %zu bytes < %zu required", ws_bytes, need);

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char *wsb = static_cast<char *>(ws);
  const size_t first = dt == AVEY_F32 ? static_cast<size_t>(B) * R * d * 4
                                      : static_cast<size_t>(B) * scale_ld(R) * 4;
  float *sc = scores ? scores : reinterpret_cast<float *>(wsb + align256(first));

  avey_status st;
  if (dt == AVEY_BF16) {
    float *inv = reinterpret_cast<float *>(wsb);
    const int ld = static_cast<int>(scale_ld(R));
    st = launch_inv_norms(static_cast<const bf16 *>(x), B, N, d, ld, inv, s);
    if (st != AVEY_OK) return st;
    if (S >= 32)
      st = launch_maxsim_pair(static_cast<const bf16 *>(x), inv, B, N, static_cast<int>(R), ld, d,
                              S, static_cast<int>(n), sc, s);
    else
      st = launch_maxsim_tc(static_cast<const bf16 *>(x), inv, B, N, static_cast<int>(R), ld, d, S,
                            static_cast<int>(n), sc, s);
  } else {
    void *xhat = wsb;
    st = launch_normalize(x, dt, B, N, d, S, xhat, s);
    if (st != AVEY_OK) return st;
    st = launch_maxsim_f32(static_cast<const float *>(xhat), B, static_cast<int>(R), d, S,
                           static_cast<int>(n), sc, s);
  }
  if (st != AVEY_OK) return st;
  return launch_topk(sc, B, static_cast<int>(n), k,
                     (flags & AVEY_RANK_UNIDIRECTIONAL) ? 1 : 0, idx, w, s);
}
