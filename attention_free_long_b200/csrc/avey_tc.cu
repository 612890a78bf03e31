// avey_tc.cu -- tcgen05 / TMEM / TMA contractions of the Avey-B hot path.
//
// Two persistent, warp-specialised kernels:
//
//   maxsim_tc_kernel (ranker, Avey-B paperlayer summary §3 and papernotes
//           整体框架), one CTA per SM: D = X_tile(128 rows) . X_tile(256 rows)^T
//           per sequence on the raw bf16 embeddings (exact products, fp32
//           accumulation); the epilogue scales each column by 1/||x_j||, takes
//           per row the max over each candidate split's S columns, scales it
//           by 1/||x_i|| (a positive factor commutes with the max), then sums
//           the maxima over the S rows of each target split.  Only the
//           [B, n, n] split scores reach HBM; neither the N x N cosines nor a
//           normalised copy of X exist.  Full grid of tiles; serves S = 16 (for
//           S >= 32 the triangular CTA-pair kernel of avey_maxsim2.cu computes
//           half the tiles).
//   layer_pair_kernel, on CTA pairs (256 x 256 tiles, cta_group::2):
//     Enricher (papernotes 整体框架, Z = sigma(XU+b); ReLU^2 per the paperlayer
//           summary App. A): D = X U with X as a bf16 split pair (two MMAs per
//           K step); epilogue scale (optional prenorm) + bias + ReLU^2, Z
//           written as a bf16 split pair.
//     Fuser (papernotes 整体框架, f = [Z_h || c] O plus residual):
//           D = [Z_h || c] O with the activation as a split pair; epilogue adds
//           the fp32 residual and writes fp32 plus the next layer's split pair.
//
// Roles (192 threads per CTA, persistent over output tiles):
//   warp 0      TMA producer: K-chunks of 64 bf16 (128-byte swizzle) of the A
//               plane(s) and B into a ring of shared-memory stages.
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators per
//               CTA) and, from one thread (of CTA 0 of a pair), issues
//               tcgen05.mma and tcgen05.commit to release stages and publish
//               accumulators.
//   warps 2-5   epilogue: tcgen05.ld of their 32 TMEM lanes (rows), fused
//               reduction / activation / residual, stores to HBM.
// The two TMEM accumulators let the epilogue of tile i overlap the MMAs of
// tile i+1.  Every barrier wait is bounded (see avey_common.cuh).
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int kEpi = 4, kThreads = 64 + 32 * kEpi;
constexpr uint32_t kTmemCols = 512;
constexpr int kRedGroups = 8, kRedCands = 16;

enum { MODE_MAXSIM = 0, MODE_ENRICH = 1, MODE_FUSE = 2 };

struct TcArgs {
  int rows;  // A rows per batch
  int cols;  // B rows (output columns)
  int kdim;  // contraction length
  int tiles_m, tiles_n, num_tiles, group_m;
  // MaxSim
  int S, n;
  float *scores;
  const float *inv_norm;  // [batch][rs_ld] 1/max(||x||, 1e-12), 0 for pad rows
  int rs_ld;
  // enricher
  const float *bias;
  const float *inv_rms;
  bf16 *out_hi;
  bf16 *out_lo;
  long long ld_out;
  // fuser: the residual is x_in (fp32) or, when x_in is null, the split pair
  // (xin_hi, xin_lo); a null x_out skips the fp32 output
  const float *x_in;
  const bf16 *xin_hi;
  const bf16 *xin_lo;
  float *x_out;
  int k_split;  // > 0: A columns >= k_split come from the second pair of maps
  // fuser: when non-null, 1 / sqrt(mean(x_out^2) + 1e-6) of every output row
  // (the next layer's prenorm scale); the pairs then walk whole row blocks
  float *rms_out;
  int *status;
};

// The j-th output tile (row block mt, column block nt) of CTA pair `pair` of
// `npairs`; false past the last.  Tiles are dealt round-robin, except when
// the fuser also writes row RMS scales: then each pair takes whole row
// blocks, all their column blocks in order, so that a row's sum of squares
// stays in one thread.
__device__ __forceinline__ bool pair_tile(const TcArgs &a, int pair, int npairs, int j, int &mt,
                                          int &nt) {
  if (a.rms_out != nullptr) {
    const int q = j / a.tiles_n;
    mt = pair + q * npairs;
    nt = j - q * a.tiles_n;
    return mt < a.tiles_m;
  }
  const long long tile = pair + static_cast<long long>(j) * npairs;
  if (tile >= a.num_tiles) return false;
  mt = static_cast<int>(tile / a.tiles_n);
  nt = static_cast<int>(tile - static_cast<long long>(mt) * a.tiles_n);
  return true;
}

// Single-CTA MaxSim: 128-row A tiles and 256-row B tiles of X.
struct MaxSimLayout {
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 4;
  static constexpr uint32_t TILES_BYTES = STAGES * STAGE_BYTES;
  static constexpr uint32_t CTRL_BYTES = 2048;  // barriers and the partial sums
  static constexpr uint32_t SMEM_BYTES = TILES_BYTES + CTRL_BYTES + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

// Decodes a MaxSim tile index into (sequence, row tile, column tile).  Groups
// of group_m row tiles walk the column tiles together so that the group's
// rows stay in L2 while every column tile streams past once.
__device__ __forceinline__ void decode_maxsim_tile(const TcArgs &a, int tile, int &b, int &mt, int &nt) {
  const int per_b = a.tiles_m * a.tiles_n;
  b = tile / per_b;
  const int local = tile - b * per_b;
  const int gsz = a.group_m * a.tiles_n;
  const int g = local / gsz;
  const int rem = local - g * gsz;
  const int rows_g = min(a.group_m, a.tiles_m - g * a.group_m);
  nt = rem / rows_g;
  mt = g * a.group_m + (rem - nt * rows_g);
}

// Time-bounded wait that ignores the abort flag (used to drain in-flight work).
__device__ __forceinline__ void mbar_wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// ---- epilogues -------------------------------------------------------------

// Per-row maxima over each candidate split's columns, summed over the rows of
// each target split inside this warp; partial sums go to red[group][cand].
template <int S>
__device__ __forceinline__ void epi_maxsim_rows(uint32_t taddr, int lane, int quarter, float *red,
                                                const float *__restrict__ col_scale,
                                                float row_scale) {
  // One 32-column TMEM chunk at a time: scale the columns by 1/||x_j||, take
  // the running row max of the candidate split, and once a candidate split is
  // complete scale by 1/||x_i|| and sum over the warp's rows.
  constexpr int CH_PER_CAND = S >= 32 ? S / 32 : 1;
  constexpr int CANDS_PER_CH = S >= 32 ? 1 : 32 / S;
  constexpr int NCH = BN / 32;
  float m[CANDS_PER_CH];
#pragma unroll 1
  for (int ch = 0; ch < NCH; ++ch) {
    const float4 *cs4 = reinterpret_cast<const float4 *>(col_scale + ch * 32);
    float4 c4[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) c4[q] = __ldg(cs4 + q);
    float v[32];
    tmem_ld32(taddr + ch * 32, v);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      v[4 * q] *= c4[q].x;
      v[4 * q + 1] *= c4[q].y;
      v[4 * q + 2] *= c4[q].z;
      v[4 * q + 3] *= c4[q].w;
    }
    if (ch % CH_PER_CAND == 0) {
#pragma unroll
      for (int u = 0; u < CANDS_PER_CH; ++u) m[u] = -INFINITY;
    }
#pragma unroll
    for (int u = 0; u < CANDS_PER_CH; ++u) {
      constexpr int W = 32 / CANDS_PER_CH;
#pragma unroll
      for (int i = 0; i < W; ++i) m[u] = fmaxf(m[u], v[u * W + i]);
    }
    if (ch % CH_PER_CAND == CH_PER_CAND - 1) {
#pragma unroll
      for (int u = 0; u < CANDS_PER_CH; ++u) {
        const int cand = (ch / CH_PER_CAND) * CANDS_PER_CH + u;
        float t = m[u] * row_scale;
        if constexpr (S >= 32) {
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
          if (lane == 0) red[quarter * kRedCands + cand] = t;
        } else {
#pragma unroll
          for (int off = 8; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
          if ((lane & 15) == 0) red[(quarter * 2 + (lane >> 4)) * kRedCands + cand] = t;
        }
      }
    }
  }
}

// Final split scores of one tile, from the per-warp partial sums.
template <int S>
__device__ __forceinline__ void epi_maxsim_write(const TcArgs &a, const float *red, int lane,
                                                 int b, int mt, int nt) {
  constexpr int TS = BM / S, NC = BN / S;
  for (int e = lane; e < TS * NC; e += 32) {
    const int ts = e / NC, cs = e - (e / NC) * NC;
    float sc = 0.f;
    if constexpr (S >= 32) {
      constexpr int per = S / 32;
#pragma unroll
      for (int q = 0; q < per; ++q) sc += red[(ts * per + q) * kRedCands + cs];
    } else {
      sc = red[ts * kRedCands + cs];
    }
    const int t = mt * TS + ts, c = nt * NC + cs;
    if (t < a.n && c < a.n) a.scores[(static_cast<long long>(b) * a.n + t) * a.n + c] = sc;
  }
}

// Output staging for TMA stores.  Each epilogue warp owns 8 KB and writes
// one 32-row x 32-column chunk at a time: row r (lane r) of an fp32 chunk is
// 128 bytes with its 16-byte pieces in the 128-byte swizzle order, a bf16
// chunk row is 64 bytes in the 64-byte swizzle order; the TMA store unswizzles
// them.  Both orders keep each shared-memory store conflict free.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }
__device__ __forceinline__ uint32_t sw64_off(int r, int c) { return r * 64 + ((c ^ ((r >> 1) & 3)) << 4); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
               : "memory");
}

// Enricher epilogue: Z = relu(scale * acc + b)^2 as a split pair, two staging
// buffers of 4 KB (hi 2 KB + lo 2 KB) alternate so that the TMA store of one
// chunk overlaps the math of the next.  `it` counts chunks across tiles.
__device__ __forceinline__ void epi_enrich(const TcArgs &a, const CUtensorMap *mhi,
                                           const CUtensorMap *mlo, uint32_t taddr, int row0,
                                           int lane, int nt, uint32_t stg, int &it) {
  const int row = row0 + lane;
  const bool valid = row < a.rows;
  const float scale = (a.inv_rms != nullptr && valid) ? a.inv_rms[row] : 1.f;
#pragma unroll 1
  for (int ch = 0; ch < BN / 32; ++ch) {
    const int col0 = nt * BN + ch * 32;
    if (col0 >= a.cols) break;  // warp-uniform
    float4 bb[8];
#pragma unroll
    for (int q = 0; q < 8; ++q)
      bb[q] = (col0 + 4 * q < a.cols) ? __ldg(reinterpret_cast<const float4 *>(a.bias + col0) + q)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    float v[32];
    tmem_ld32(taddr + ch * 32, v);
    const uint32_t buf = stg + (it & 1) * 4096;
    if (it >= 2) {  // the store issued from this buffer two chunks ago must have read it
      if (lane == 0) bulk_wait_read<1>();
      __syncwarp();
    }
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float b4[4] = {bb[q].x, bb[q].y, bb[q].z, bb[q].w};
#pragma unroll
      for (int j = 0; j < 4; j += 2) {
        float z0 = fmaxf(fmaf(v[4 * q + j], scale, b4[j]), 0.f);
        float z1 = fmaxf(fmaf(v[4 * q + j + 1], scale, b4[j + 1]), 0.f);
        split_pack(z0 * z0, z1 * z1, hi[2 * q + j / 2], lo[2 * q + j / 2]);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      st_shared_v4(buf + sw64_off(lane, c), hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
      st_shared_v4(buf + 2048 + sw64_off(lane, c), lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(mhi, buf, col0, row0, 0);
      tma_store_3d(mlo, buf + 2048, col0, row0, 0);
      bulk_commit();
    }
    (void)valid;
    ++it;
  }
}

// The residual of one row's 32-column chunk as raw 16-byte words, zeros
// outside the matrix: eight words of the fp32 x_in, or four words of each
// plane of its split pair.  fuse_residual_values turns them into fp32 where
// they are used, so that the loads stay in flight until then.
__device__ __forceinline__ void fuse_load_residual(const TcArgs &a, int row, int col0, uint4 (&r)[8]) {
  const bool valid = row < a.rows;
  const long long off = static_cast<long long>(row) * a.cols + col0;
  const uint4 zero = make_uint4(0, 0, 0, 0);
  if (a.x_in != nullptr) {
    const uint4 *src = reinterpret_cast<const uint4 *>(a.x_in + off);
#pragma unroll
    for (int q = 0; q < 8; ++q) r[q] = (valid && col0 + 4 * q < a.cols) ? src[q] : zero;
  } else {
    const uint4 *h = reinterpret_cast<const uint4 *>(a.xin_hi + off);
    const uint4 *l = reinterpret_cast<const uint4 *>(a.xin_lo + off);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const bool ok = valid && col0 + 8 * q < a.cols;
      r[q] = ok ? h[q] : zero;
      r[4 + q] = ok ? l[q] : zero;
    }
  }
}
// hi + lo of two bf16 is exact in fp32 (the lo part sits at least 8 bits below hi).
__device__ __forceinline__ void fuse_residual_values(const TcArgs &a, const uint4 (&r)[8], float (&x)[32]) {
  if (a.x_in != nullptr) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      x[4 * q] = __uint_as_float(r[q].x);
      x[4 * q + 1] = __uint_as_float(r[q].y);
      x[4 * q + 2] = __uint_as_float(r[q].z);
      x[4 * q + 3] = __uint_as_float(r[q].w);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t hw[4] = {r[q].x, r[q].y, r[q].z, r[q].w};
      const uint32_t lw[4] = {r[4 + q].x, r[4 + q].y, r[4 + q].z, r[4 + q].w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 h = unpack_bf16(hw[u]), l = unpack_bf16(lw[u]);
        x[8 * q + 2 * u] = h.x + l.x;
        x[8 * q + 2 * u + 1] = h.y + l.y;
      }
    }
  }
}

// Fuser epilogue: x_out = x_in + acc (fp32) and/or its split pair; one 8 KB
// staging buffer (fp32 4 KB, hi 2 KB, lo 2 KB).  The residuals of chunks 0
// and 1 arrive requested (xi, xj, issued before the accumulator wait); each
// chunk issues the loads of the chunk two ahead before its own math, so two
// chunks' loads are always in flight behind it.
__device__ __forceinline__ void epi_fuse(const TcArgs &a, const CUtensorMap *mout,
                                         const CUtensorMap *mhi, const CUtensorMap *mlo,
                                         uint32_t taddr, int row0, int lane, int nt, uint32_t stg,
                                         int &it, uint4 (&xi)[8], uint4 (&xj)[8], float &ss) {
  const int row = row0 + lane;
  const bool pair = a.out_hi != nullptr;
  const bool f32out = a.x_out != nullptr;
#pragma unroll 1
  for (int ch = 0; ch < BN / 32; ++ch) {
    const int col0 = nt * BN + ch * 32;
    if (col0 >= a.cols) break;  // warp-uniform
    uint4 xn[8];
    if (ch + 2 < BN / 32) fuse_load_residual(a, row, col0 + 64, xn);
    float v[32];
    tmem_ld32(taddr + ch * 32, v);
    if (it >= 1) {  // the previous chunk's stores must have read the buffer
      if (lane == 0) bulk_wait_read<0>();
      __syncwarp();
    }
    float o[32];
    fuse_residual_values(a, xi, o);
#pragma unroll
    for (int q = 0; q < 32; ++q) o[q] += v[q];
    if (a.rms_out != nullptr) {
#pragma unroll
      for (int q = 0; q < 32; ++q) ss = fmaf(o[q], o[q], ss);
    }
    if (f32out) {
#pragma unroll
      for (int c = 0; c < 8; ++c)
        st_shared_v4(stg + sw128_off(lane, c), __float_as_uint(o[4 * c]), __float_as_uint(o[4 * c + 1]),
                     __float_as_uint(o[4 * c + 2]), __float_as_uint(o[4 * c + 3]));
    }
    if (pair) {
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) split_pack(o[2 * j], o[2 * j + 1], hi[j], lo[j]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        st_shared_v4(stg + 4096 + sw64_off(lane, c), hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
        st_shared_v4(stg + 6144 + sw64_off(lane, c), lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
      }
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      if (f32out) tma_store_3d(mout, stg, col0, row0, 0);
      if (pair) {
        tma_store_3d(mhi, stg + 4096, col0, row0, 0);
        tma_store_3d(mlo, stg + 6144, col0, row0, 0);
      }
      bulk_commit();
    }
    ++it;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      xi[q] = xj[q];
      xj[q] = xn[q];
    }
  }
}

// ---- single-CTA MaxSim ------------------------------------------------------

template <int SPLIT_S>
__global__ void __launch_bounds__(kThreads, 1)
    maxsim_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const TcArgs a) {
  using L = MaxSimLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t *ctrl = smem_raw + pad + L::TILES_BYTES;
  const uint32_t sbase = raw_s + pad;
  const uint32_t cbase = sbase + L::TILES_BYTES;
  static_assert(L::STAGES <= 8, "the control block holds at most 8 stages");
  // control block: full[8] @0, empty[8] @64, tfull[2] @128, tempty[2] @144,
  // redbar[2 acc] @160, drain @192, tmem base @200, abort flag @204,
  // partial sums [2 acc][8 groups][16 candidates] @256
  auto full_bar = [&](int s) { return cbase + 8u * s; };
  auto empty_bar = [&](int s) { return cbase + 64u + 8u * s; };
  auto tfull_bar = [&](int i) { return cbase + 128u + 8u * i; };
  auto tempty_bar = [&](int i) { return cbase + 144u + 8u * i; };
  auto red_bar = [&](int i) { return cbase + 160u + 8u * i; };
  const uint32_t drain_bar = cbase + 192u;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(ctrl + 200);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 204);
  float *red = reinterpret_cast<float *>(ctrl + 256);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), kEpi);
    }
    for (int i = 0; i < 2; ++i) mbar_init(red_bar(i), 4);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(ctrl + 200), kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int kchunks = (a.kdim + BK - 1) / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        int b, mt, nt;
        decode_maxsim_tile(a, tile, b, mt, nt);
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + stage * L::STAGE_BYTES;
          mbar_arrive_expect_tx(full_bar(stage), L::STAGE_BYTES);
          tma_load_3d(st, &tmA, full_bar(stage), kc * BK, mt * BM, b);
          tma_load_3d(st + L::A_BYTES, &tmB, full_bar(stage), kc * BK, nt * BN, b);
          ++issued;
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      // Drain: every load issued must land before the CTA may exit.
      for (int s = 0; s < L::STAGES; ++s) {
        if (issued > s) {
          const long long last = ((issued - 1 - s) / L::STAGES) * L::STAGES + s;
          mbar_wait_drain(full_bar(s), static_cast<uint32_t>((last / L::STAGES) & 1));
        }
      }
    }
  } else if (warp == 1) {
    // ----------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(BM, BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + stage * L::STAGE_BYTES;
          const uint64_t da = sdesc_k_sw128(st);
          const uint64_t db = sdesc_k_sw128(st + L::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // +32 bytes along K inside the 128-byte swizzled row = +2 in the
            // descriptor's 16-byte address units.
            tc_mma_bf16(d_tmem, da + 2u * kk, db + 2u * kk, idesc, (kc | kk) != 0);
          }
          tc_commit(empty_bar(stage));
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(tfull_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      int b, mt, nt;
      decode_maxsim_tile(a, tile, b, mt, nt);
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quarter * 32) << 16);
      const int row = mt * BM + quarter * 32 + lane;
      float *red_acc = red + acc * kRedGroups * kRedCands;
      const float *rs = a.inv_norm + static_cast<long long>(b) * a.rs_ld;
      epi_maxsim_rows<SPLIT_S>(taddr, lane, quarter, red_acc, rs + nt * BN, rs[row]);
      __syncwarp();
      if (lane == 0) mbar_arrive(red_bar(acc));
      if (warp == 2) {
        // leader warp: combine the four warps' partial sums
        if (!mbar_wait(red_bar(acc), acc_phase, abort_flag)) {
          ok = false;
        } else {
          epi_maxsim_write<SPLIT_S>(a, red_acc, lane, b, mt, nt);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
      if (!ok) break;
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (!ok) {
      *abort_flag = 1;
      record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ---- layer GEMMs on CTA pairs ------------------------------------------------
//
// The enricher and the fuser on clusters of two CTAs (tcgen05 cta_group::2):
// a pair owns a 256 x 256 output tile.  Each CTA keeps 128 of its rows in
// TMEM, loads those rows of both activation planes and one 128-row half of
// the weight tile, and CTA 0 issues M = 256, N = 256, K = 16 MMAs that read
// the activation rows and both weight halves across the pair.  Per FLOP each
// SM moves a quarter fewer operand bytes from L2 than with 128 x 256 tiles on
// one SM, and four 48 KB stages cover a third more load latency than three
// of 64 KB.  The epilogues are the single-CTA ones, each CTA on its own rows.
//
// Barriers: both CTAs' loads complete on CTA 0's "full" barrier; the MMA
// commit frees the stage in both CTAs and publishes the accumulator to both;
// both CTAs' epilogue warps release the accumulator to CTA 0.  Every load
// fills only the issuing CTA's own shared memory.

struct PairLayout {
  static constexpr int PM = 256;                        // rows per pair tile
  static constexpr uint32_t A_BYTES = 128 * BK * 2;     // one plane, this CTA's rows
  static constexpr uint32_t B_BYTES = 128 * BK * 2;     // this CTA's half of the weight tile
  static constexpr uint32_t STAGE_BYTES = 2 * A_BYTES + B_BYTES;
  static constexpr int STAGES = 4;
  static constexpr uint32_t TILES_BYTES = STAGES * STAGE_BYTES;
  static constexpr uint32_t CTRL_BYTES = 1024;
  static constexpr uint32_t STAGING_BYTES = kEpi * 8192;
  static constexpr uint32_t SMEM_BYTES = TILES_BYTES + CTRL_BYTES + STAGING_BYTES + 1024;
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(STAGES <= 8, "the control block holds at most 8 stages");
};

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    layer_pair_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                      const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmO0,
                      const __grid_constant__ CUtensorMap tmO1, const __grid_constant__ CUtensorMap tmO2,
                      const __grid_constant__ CUtensorMap tmC0, const __grid_constant__ CUtensorMap tmC1,
                      const TcArgs a) {
  static_assert(MODE == MODE_ENRICH || MODE == MODE_FUSE, "layer GEMMs only");
  using P = PairLayout;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t *ctrl = smem_raw + pad + P::TILES_BYTES;
  const uint32_t sbase = raw_s + pad;
  const uint32_t cbase = sbase + P::TILES_BYTES;
  // control block: full[8] @0, empty[8] @64, tfull[2] @128, tempty[2] @144,
  // drain @160, tmem base @168, abort flag @172
  auto full_bar = [&](int s) { return cbase + 8u * s; };
  auto empty_bar = [&](int s) { return cbase + 64u + 8u * s; };
  auto tfull_bar = [&](int i) { return cbase + 128u + 8u * i; };
  auto tempty_bar = [&](int i) { return cbase + 144u + 8u * i; };
  const uint32_t drain_bar = cbase + 160u;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(ctrl + 168);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 172);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 2 * kEpi);  // both CTAs' epilogue warps (used in CTA 0)
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA0);
    prefetch_tmap(&tmA1);
    prefetch_tmap(&tmB);
    prefetch_tmap(&tmO0);
    prefetch_tmap(&tmO1);
    if (MODE == MODE_FUSE) prefetch_tmap(&tmO2);
    if (MODE == MODE_FUSE && a.k_split > 0) {
      prefetch_tmap(&tmC0);
      prefetch_tmap(&tmC1);
    }
  }
  cluster_sync_all();  // barriers of both CTAs initialised before any remote use
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(ctrl + 168), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int kchunks = (a.kdim + BK - 1) / BK;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      int mt, nt;
      for (int j = 0; ok && pair_tile(a, pair, npairs, j, mt, nt); ++j) {
        const int arow = mt * P::PM + static_cast<int>(rank) * 128;
        const int brow = nt * BN + static_cast<int>(rank) * 128;
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * P::STAGE_BYTES);
          const uint32_t full0 = mapa_shared(full_bar(stage), 0);
          const uint32_t st = sbase + stage * P::STAGE_BYTES;
          // fuser with a separate contextualizer output: [Z_h || c] from two
          // sources, split at a multiple of the K chunk
          const bool from_c = MODE == MODE_FUSE && a.k_split > 0 && kc * BK >= a.k_split;
          const CUtensorMap *ma = from_c ? &tmC0 : &tmA0;
          const CUtensorMap *mal = from_c ? &tmC1 : &tmA1;
          const int ax = from_c ? kc * BK - a.k_split : kc * BK;
          tma_load_3d_pair(st, ma, full0, ax, arow, 0);
          tma_load_3d_pair(st + P::A_BYTES, mal, full0, ax, arow, 0);
          tma_load_3d_pair(st + 2 * P::A_BYTES, &tmB, full0, kc * BK, brow, 0);
          ++issued;
          if (++stage == P::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      // Drain: the pair's MMA has consumed (so the loads have landed in) every
      // stage this CTA filled once its last use is released.
      for (int s = 0; s < P::STAGES; ++s) {
        if (issued > s) {
          const long long last = ((issued - 1 - s) / P::STAGES) * P::STAGES + s;
          mbar_wait_drain(empty_bar(s), static_cast<uint32_t>((last / P::STAGES) & 1));
        }
      }
    }
  } else if (warp == 1) {
    // --------------------------------------------------- MMA issue (CTA 0)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(P::PM, BN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int mt_, nt_;
      for (int jt = 0; ok && pair_tile(a, pair, npairs, jt, mt_, nt_); ++jt) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + stage * P::STAGE_BYTES;
          const uint64_t da0 = sdesc_k_sw128(st);
          const uint64_t da1 = sdesc_k_sw128(st + P::A_BYTES);
          const uint64_t db = sdesc_k_sw128(st + 2 * P::A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            tc_mma_bf16_pair(d_tmem, da0 + 2u * kk, db + 2u * kk, idesc, (kc | kk) != 0);
            tc_mma_bf16_pair(d_tmem, da1 + 2u * kk, db + 2u * kk, idesc, 1u);
          }
          tc_commit_pair_both(empty_bar(stage));
          if (++stage == P::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_both(tfull_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      tc_commit_pair_both(drain_bar);
      mbar_wait_drain(drain_bar, 0);
    }
  } else {
    // ------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    const uint32_t stg = cbase + P::CTRL_BYTES + static_cast<uint32_t>(warp - 2) * 8192u;
    const uint32_t tempty_r0 = mapa_shared(tempty_bar(0), 0), tempty_r1 = mapa_shared(tempty_bar(1), 0);
    int acc = 0, it = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    float ss = 0.f;  // fuser with row RMS output: this row's sum of squares so far
    int mt, nt;
    for (int j = 0; pair_tile(a, pair, npairs, j, mt, nt); ++j) {
      const int row0 = mt * P::PM + static_cast<int>(rank) * 128 + quarter * 32;
      uint4 xi[8], xj[8];
      if constexpr (MODE == MODE_FUSE) {
        fuse_load_residual(a, row0 + lane, nt * BN, xi);
        fuse_load_residual(a, row0 + lane, nt * BN + 32, xj);
      }
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + static_cast<uint32_t>(acc * BN) + (static_cast<uint32_t>(quarter * 32) << 16);
      if constexpr (MODE == MODE_ENRICH) {
        epi_enrich(a, &tmO0, &tmO1, taddr, row0, lane, nt, stg, it);
      } else {
        if (nt == 0) ss = 0.f;
        epi_fuse(a, &tmO0, &tmO1, &tmO2, taddr, row0, lane, nt, stg, it, xi, xj, ss);
        if (a.rms_out != nullptr && nt == a.tiles_n - 1 && row0 + lane < a.rows)
          a.rms_out[row0 + lane] = 1.0f / sqrtf(ss / static_cast<float>(a.cols) + 1e-6f);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_r1 : tempty_r0);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (!ok) {
      *abort_flag = 1;
      record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
    }
    if (lane == 0) bulk_wait_all();  // outputs written
  }

  tc_fence_before();
  __syncthreads();
  // Both CTAs past their loops: the pair's MMAs have drained (CTA 0 waited on
  // the drain commit) and no remote arrival is still on its way.
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
  cluster_sync_all();
}

template <int MODE>
avey_status run_layer_pair(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b,
                           const CUtensorMap &o0, const CUtensorMap &o1, const CUtensorMap &o2,
                           const CUtensorMap &c0, const CUtensorMap &c1, TcArgs args, cudaStream_t st,
                           const char *name) {
  using P = PairLayout;
  if (args.num_tiles <= 0) return AVEY_OK;
  auto kern = layer_pair_kernel<MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(P::SMEM_BYTES));
  if (e != cudaSuccess) {
    set_detail("%s: cudaFuncSetAttribute: %s", name, cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  // Persistent grid: as many pairs as can be resident at once (a pair needs
  // two SMs of one GPC, so this can be below half the SM count).
  static int resident[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int &cap = resident[dev & 63];
  if (cap == 0) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * (sm_count() / 2));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = P::SMEM_BYTES;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess || clusters < 1) {
      set_detail("%s: no resident CTA pair (%s)", name, cudaGetErrorString(e));
      return AVEY_ERR_CUDA;
    }
    cap = std::min(clusters, sm_count() / 2);
  }
  const int pairs = std::max(1, std::min(args.num_tiles, cap));
  kern<<<2 * pairs, kThreads, P::SMEM_BYTES, st>>>(a0, a1, b, o0, o1, o2, c0, c1, args);
  AVEY_CHECK_LAUNCH(name, st);
  return AVEY_OK;
}

template <int SPLIT_S>
avey_status run_maxsim_tc(const CUtensorMap &ma, const CUtensorMap &mb, TcArgs args, cudaStream_t st) {
  using L = MaxSimLayout;
  if (args.num_tiles <= 0) return AVEY_OK;
  auto kern = maxsim_tc_kernel<SPLIT_S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::SMEM_BYTES));
  if (e != cudaSuccess) {
    set_detail("maxsim_tc: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  const int grid = std::min(args.num_tiles, sm_count());
  kern<<<grid, kThreads, L::SMEM_BYTES, st>>>(ma, mb, args);
  AVEY_CHECK_LAUNCH("maxsim_tc", st);
  return AVEY_OK;
}

TcArgs base_args(int rows, int cols, int kdim) {
  TcArgs a{};
  a.rows = rows;
  a.cols = cols;
  a.kdim = kdim;
  a.tiles_m = (rows + BM - 1) / BM;
  a.tiles_n = (cols + BN - 1) / BN;
  a.num_tiles = a.tiles_m * a.tiles_n;
  a.group_m = 1;
  a.status = device_status_word();
  return a;
}

// Pair tiles: 256 rows (two CTAs of 128) x 256 output columns.
TcArgs pair_args(int rows, int cols, int kdim) {
  TcArgs a = base_args(rows, cols, kdim);
  a.tiles_m = (rows + PairLayout::PM - 1) / PairLayout::PM;
  a.num_tiles = a.tiles_m * a.tiles_n;
  return a;
}

}  // namespace

avey_status launch_maxsim_tc(const bf16 *x, const float *inv_norm, int B, int N, int R, int rs_ld,
                             int d, int S, int n, float *scores, cudaStream_t s) {
  // The maps cover the unpadded [B, N, d] embeddings: rows N..R-1 of the last
  // split (and any tile rows past R) read as zeros, which is the padding.
  CUtensorMap ma, mb;
  const uint64_t rs = static_cast<uint64_t>(d) * 2, bs = rs * static_cast<uint64_t>(N);
  if (!encode_bf16_map(&ma, x, d, N, B, rs, bs, BM)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&mb, x, d, N, B, rs, bs, BN)) return AVEY_ERR_CUDA;
  TcArgs a = base_args(R, R, d);
  a.num_tiles = a.tiles_m * a.tiles_n * B;
  a.group_m = 16;
  a.S = S;
  a.n = n;
  a.scores = scores;
  a.inv_norm = inv_norm;
  a.rs_ld = rs_ld;
  switch (S) {
    case 16: return run_maxsim_tc<16>(ma, mb, a, s);
    default:
      set_detail("maxsim_tc: S=%d unsupported (16; larger splits use the CTA-pair kernel)", S);
      return AVEY_ERR_UNSUPPORTED;
  }
}

avey_status launch_enrich_tc(const bf16 *xhi, const bf16 *xlo, int T, int d, const bf16 *Ut,
                             int m, const float *bias, const float *inv_rms, bf16 *zhi,
                             bf16 *zlo, cudaStream_t s) {
  CUtensorMap a0, a1, mb, o0, o1;
  const uint64_t rs = static_cast<uint64_t>(d) * 2, zs = static_cast<uint64_t>(m) * 2;
  if (!encode_bf16_map(&a0, xhi, d, T, 1, rs, rs * T, BM)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&a1, xlo, d, T, 1, rs, rs * T, BM)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&mb, Ut, d, m, 1, rs, rs * m, 128)) return AVEY_ERR_CUDA;
  if (!encode_map(&o0, false, zhi, m, T, 1, zs, zs * T, 32, 32, 64)) return AVEY_ERR_CUDA;
  if (!encode_map(&o1, false, zlo, m, T, 1, zs, zs * T, 32, 32, 64)) return AVEY_ERR_CUDA;
  TcArgs a = pair_args(T, m, d);
  a.bias = bias;
  a.inv_rms = inv_rms;
  a.out_hi = zhi;
  a.out_lo = zlo;
  a.ld_out = m;
  return run_layer_pair<MODE_ENRICH>(a0, a1, mb, o0, o1, o1, a0, a1, a, s, "enrich_tc");
}

avey_status launch_fuse_tc(const bf16 *ahi, const bf16 *alo, int T, int m, const bf16 *Ot, int d,
                           const float *x_in, const bf16 *xin_hi, const bf16 *xin_lo, float *x_out,
                           bf16 *xo_hi, bf16 *xo_lo, cudaStream_t s, const bf16 *chi,
                           const bf16 *clo, int k_split, float *rms_out) {
  if ((x_in == nullptr && (xin_hi == nullptr || xin_lo == nullptr)) ||
      (x_out == nullptr && xo_hi == nullptr)) {
    set_detail("fuse_tc: needs a residual (fp32 or pair) and an output (fp32 or pair)");
    return AVEY_ERR_INVALID_ARG;
  }
  CUtensorMap a0, a1, mb, o0, o1, o2, c0, c1;
  const uint64_t rs = static_cast<uint64_t>(m) * 2;
  const uint64_t fs = static_cast<uint64_t>(d) * 4, hs = static_cast<uint64_t>(d) * 2;
  if (!encode_bf16_map(&a0, ahi, m, T, 1, rs, rs * T, BM)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&a1, alo, m, T, 1, rs, rs * T, BM)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&mb, Ot, m, d, 1, rs, rs * d, 128)) return AVEY_ERR_CUDA;
  if (x_out != nullptr && !encode_map(&o0, true, x_out, d, T, 1, fs, fs * T, 32, 32, 128))
    return AVEY_ERR_CUDA;
  if (xo_hi != nullptr) {
    if (!encode_map(&o1, false, xo_hi, d, T, 1, hs, hs * T, 32, 32, 64)) return AVEY_ERR_CUDA;
    if (!encode_map(&o2, false, xo_lo, d, T, 1, hs, hs * T, 32, 32, 64)) return AVEY_ERR_CUDA;
  }
  // the kernel never uses the map of an output it does not write
  if (x_out == nullptr) o0 = o1;
  if (xo_hi == nullptr) o1 = o2 = o0;
  TcArgs a = pair_args(T, d, m);
  a.x_in = x_in;
  a.xin_hi = xin_hi;
  a.xin_lo = xin_lo;
  a.x_out = x_out;
  a.out_hi = xo_hi;
  a.out_lo = xo_lo;
  a.ld_out = d;
  a.rms_out = rms_out;
  if (chi != nullptr) {
    // columns [k_split, m) of the activation come from c [T, m - k_split]
    if (k_split <= 0 || k_split % BK != 0 || k_split >= m) {
      set_detail("fuse_tc: split at %d must be a positive multiple of %d below m = %d", k_split, BK, m);
      return AVEY_ERR_INVALID_ARG;
    }
    const uint64_t cs = static_cast<uint64_t>(m - k_split) * 2;
    if (!encode_bf16_map(&c0, chi, m - k_split, T, 1, cs, cs * T, BM)) return AVEY_ERR_CUDA;
    if (!encode_bf16_map(&c1, clo, m - k_split, T, 1, cs, cs * T, BM)) return AVEY_ERR_CUDA;
    a.k_split = k_split;
    return run_layer_pair<MODE_FUSE>(a0, a1, mb, o0, o1, o2, c0, c1, a, s, "fuse_tc");
  }
  return run_layer_pair<MODE_FUSE>(a0, a1, mb, o0, o1, o2, a0, a1, a, s, "fuse_tc");
}

}  // namespace avey
