// avey_compress_tc.cu -- neural compression with residual on tcgen05, S = 64
// or 128 (papernotes 关键设计 4, eq. 8; paperlayer summary §4.3, App. H):
//   out(t) = sum_{r=0..k} w_r P_r X_{c_r} + X_t,   c_0 = t, w_0 = 1.
//
// A tile is (target split t, 128-feature slab); per retrieved block r the
// tensor cores compute the transposed partial product
//   D_r[f, i] = sum_j X_{c_r}[j, f] P[i, rS + j]     (M = 128 f, N = S i, K = S j)
// with the block's S token rows gathered by TMA straight from the token-major
// embeddings (an MN-major A operand: boxes of 64 features x S tokens, 128-byte
// swizzle) and P_r as the K-major B operand (S / 64 boxes of 64 j).  Every D_r
// lands in its own TMEM buffer of S columns; the epilogue (thread = feature f)
// adds w_r D_r into fp32 registers, so the weight multiplies the fp32 product
// and the bf16 inputs are never re-rounded; block 0 also accumulates X_t^T I
// (the residual, exact, against a 64 x 64 identity per 64 tokens), and the
// epilogue writes fp32 and/or the split pair straight to global memory (per
// token, the warp's 32 lanes store 32 consecutive features), so that all of
// shared memory but the identity (and, for S = 64 with k + 1 <= 8, all of P,
// 64 KB, loaded once) goes to the ring of loads.  A stage holds a group of
// consecutive present blocks of one tile, two for S = 64 and one for S = 128:
// the single MMA-issuing thread pays a fixed cost per stage (its waits, fence,
// first MMA and commits) that exceeds the tensor time of a 16 KB block, so a
// pair of blocks per stage halves it.  Four stages of 32 KB (X alone) for
// S = 64 with P resident, else four of 48 KB; three of 64 KB for S = 128.
// Roles: warp 0 TMA producer, warp 1 TMEM allocation and MMA issue, warps 2-9
// epilogue (two per TMEM lane quarter = 32 features, each on half of the
// split's S tokens).  Every wait is bounded.
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

constexpr int CF = 128;                       // features per tile (M)
constexpr int C_EPI = 8, C_THR = 64 + 32 * C_EPI;
constexpr uint32_t C_IDENT = 64 * 64 * 2;     // 8 KB: the 64 x 64 identity (B operand)

template <int S, int KM>
struct CompLayout {
  static_assert(S == 64 || S == 128, "split size");
  static constexpr uint32_t XBOX = 64 * S * 2;   // 64 features x S tokens
  static constexpr uint32_t XB = 2 * XBOX;       // the block's 128-feature slab
  static constexpr int PCH = S / 64;             // K chunks of P_r, 64 j each
  static constexpr uint32_t PBOX = S * 64 * 2;   // S i x 64 j
  // For S = 64 and k + 1 <= 8, all of P (64 KB) stays in shared memory for
  // the whole launch and the ring carries X alone; otherwise every stage also
  // carries its block's P_r.
  static constexpr bool PRES = S == 64 && KM == 8;
  static constexpr uint32_t PRES_BYTES = PRES ? KM * PBOX : 0;
  // A stage holds a group of G consecutive present blocks of one tile (the
  // last group of a tile may hold fewer): every per-stage cost of the single
  // MMA-issuing thread (its waits, fence and commits) is paid once per group.
  // S = 128 blocks are too large for two per stage.
  static constexpr int G = S == 64 ? 2 : 1;
  static constexpr uint32_t SLOT = XB + (PRES ? 0 : PCH * PBOX);  // one block of a stage
  static constexpr uint32_t STAGE = G * SLOT;
  static constexpr int STAGES = S == 64 ? 4 : 3;
  static constexpr int NACC = 512 / S;           // TMEM buffers of S columns
  static constexpr int NGRP = NACC / G;          // groups of buffers in flight
  static constexpr int TOK = S / 2;              // tokens per epilogue warp
  // barriers and flags in the first 512 bytes, then two block lists of KM (split, weight)
  static constexpr uint32_t CTRL = (512 + 2 * KM * 8 + 1023) / 1024 * 1024;
  static constexpr uint32_t SMEM = STAGES * STAGE + PRES_BYTES + C_IDENT + CTRL + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(STAGES <= 16 && NACC <= 8, "the control block holds 16 stages and 8 buffers");
  static_assert(G == 1 || TOK == 32, "the epilogue reads a pair of blocks with one wait");
};

struct CompArgs {
  int N, d, n, k, nslab, num_tiles;
  int t0, nr;  // targets t0 .. t0+nr-1 of every sequence; idx, w, out are [B, nr, ...]
  const int32_t *idx;
  const float *w;
  const bf16 *x;
  float *out;
  bf16 *out_hi, *out_lo;
  int *status;
};

__device__ __forceinline__ uint64_t cdesc_k(uint32_t a) {
  return static_cast<uint64_t>((a >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1u) << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
         (static_cast<uint64_t>(2u) << 61);
}
// MN-major, 128-byte swizzle: 64 features per 128-byte row (one row per
// token), 8-token atoms 1024 bytes apart, the two 64-feature groups `group`
// bytes apart.
__device__ __forceinline__ uint64_t cdesc_mn(uint32_t a, uint32_t group) {
  return static_cast<uint64_t>((a >> 4) & 0x3FFFu) | (static_cast<uint64_t>(group >> 4) << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
         (static_cast<uint64_t>(2u) << 61);
}

__device__ __forceinline__ void cwait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// The block list of one tile (target t = tile's split, local row seg = b*nr +
// t - t0 of idx / w): split c[r] and weight wr[r] of block r <= k, c[0] = t,
// w[0] = 1, c = -1 for no block.  load_list only issues the loads (so that
// they can be in flight one tile ahead); check_list turns out-of-range indices
// into -1 and records them.  KM >= k + 1 keeps the list in registers.
template <int KM>
__device__ __forceinline__ void load_list(const CompArgs &a, int tile, int (&c)[KM], float (&wr)[KM]) {
  const long long seg = tile / a.nslab;
  const int b = static_cast<int>(seg / a.nr);
  c[0] = a.t0 + static_cast<int>(seg - static_cast<long long>(b) * a.nr);
  wr[0] = 1.f;
#pragma unroll
  for (int r = 1; r < KM; ++r) {
    c[r] = -1;
    wr[r] = 0.f;
    if (r <= a.k) {
      c[r] = __ldg(a.idx + seg * a.k + (r - 1));
      wr[r] = __ldg(a.w + seg * a.k + (r - 1));
    }
  }
}
template <int KM>
__device__ __forceinline__ void check_list(const CompArgs &a, int (&c)[KM]) {
#pragma unroll
  for (int r = 1; r < KM; ++r) {
    if (c[r] < -1 || c[r] >= a.n) {
      record_status(a.status, AVEY_ERR_DEVICE_BOUNDS);
      c[r] = -1;
    }
  }
}

template <int S, int KM>
__global__ void __launch_bounds__(C_THR, 1)
    compress_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                       const CompArgs a) {
  using L = CompLayout<S, KM>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t *ident = smem_raw + pad + L::STAGES * L::STAGE + L::PRES_BYTES;
  uint8_t *ctrl = ident + C_IDENT;
  const uint32_t sbase = raw_s + pad;
  const uint32_t pbase = sbase + L::STAGES * L::STAGE;  // resident P (PRES)
  const uint32_t ibase = pbase + L::PRES_BYTES;
  const uint32_t cbase = ibase + C_IDENT;
  // control block: full[16] @0, empty[16] @128, tfull[8] @256, tempty[8]
  // @320, drain @384, tmem base @392, abort flag @396, lfull[2] @400,
  // lempty[2] @416, pready @432, block lists [2][KM] of (split, weight) @512
  static_assert(512 + 2 * KM * 8 <= L::CTRL, "the block lists fit the control block");
  auto full_bar = [&](int s) { return cbase + 8u * s; };
  auto empty_bar = [&](int s) { return cbase + 128u + 8u * s; };
  auto tfull_bar = [&](int i) { return cbase + 256u + 8u * i; };
  auto tempty_bar = [&](int i) { return cbase + 320u + 8u * i; };
  const uint32_t drain_bar = cbase + 384u;
  auto lfull_bar = [&](int i) { return cbase + 400u + 8u * i; };
  auto lempty_bar = [&](int i) { return cbase + 416u + 8u * i; };
  const uint32_t pready_bar = cbase + 432u;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(ctrl + 392);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 396);
  int *list_c = reinterpret_cast<int *>(ctrl + 512);               // [2][KM]
  float *list_w = reinterpret_cast<float *>(ctrl + 512 + 2 * KM * 4);  // [2][KM]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < L::NGRP; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), C_EPI);
    }
    mbar_init(drain_bar, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(lfull_bar(i), 1);
      mbar_init(lempty_bar(i), 1 + C_EPI);  // the MMA issuer and the epilogue warps
    }
    mbar_init(pready_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(ctrl + 392), 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmP);
  }
  // The residual X_t enters block 0's accumulator through the tensor cores:
  // D_0 += X_t^T I with I the 64 x 64 identity, a K-major B operand in the
  // 128-byte-swizzled layout (row i = 64 bf16; its 16-byte chunk q sits at
  // chunk q ^ (i & 7)), once per 64 tokens.  Products with 1 and 0 are exact,
  // so D_0 gains X_t exactly, in fp32.
  for (int e = threadIdx.x; e < static_cast<int>(C_IDENT / 16); e += C_THR)
    reinterpret_cast<uint4 *>(ident)[e] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (threadIdx.x < 64) {
    const int i = threadIdx.x;
    const int chunk = (i >> 3) ^ (i & 7);
    reinterpret_cast<bf16 *>(ident + i * 128 + chunk * 16)[i & 7] = __float2bfloat16_rn(1.f);
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // -------------------------------------------------------------- producer
    // Loads each tile's block list one tile ahead, publishes it in a shared
    // slot for the MMA issuer and the epilogue, then gathers its blocks.
    if (lane == 0) {
      int stage = 0, it = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      if constexpr (L::PRES) {  // P_0 .. P_k, once for the launch
        mbar_arrive_expect_tx(pready_bar, static_cast<uint32_t>(a.k + 1) * L::PBOX);
        for (int r = 0; r <= a.k; ++r)
          tma_load_3d(pbase + r * L::PBOX, &tmP, pready_bar, r * S, 0, 0);
      }
      int cn[KM];
      float wn[KM];
      if (static_cast<int>(blockIdx.x) < a.num_tiles) load_list<KM>(a, blockIdx.x, cn, wn);
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x, ++it) {
        const long long seg = tile / a.nslab;  // b * nr + (t - t0)
        const int slab = static_cast<int>(tile - seg * a.nslab);
        const int b = static_cast<int>(seg / a.nr);
        int cl[KM];
        float wl[KM];
#pragma unroll
        for (int r = 0; r < KM; ++r) {
          cl[r] = cn[r];
          wl[r] = wn[r];
        }
        if (tile + static_cast<int>(gridDim.x) < a.num_tiles)
          load_list<KM>(a, tile + gridDim.x, cn, wn);  // in flight during this tile
        check_list<KM>(a, cl);
        const int slot = it & 1;
        if (!mbar_wait(lempty_bar(slot), ((it >> 1) & 1) ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
#pragma unroll
        for (int r = 0; r < KM; ++r) {
          list_c[slot * KM + r] = cl[r];
          list_w[slot * KM + r] = wl[r];
        }
        mbar_arrive(lfull_bar(slot));
        uint64_t left = 0;  // the tile's present blocks (k + 1 <= 33)
#pragma unroll
        for (int r = 0; r < KM; ++r) left |= (cl[r] >= 0 ? 1ull : 0ull) << r;
#pragma unroll 1
        while (left != 0u) {
          // the next group: up to G present blocks in rank order
          int rg[L::G];
          int nb = 0;
#pragma unroll
          for (int j = 0; j < L::G; ++j) {
            rg[j] = -1;
            if (left != 0u) {
              rg[j] = __ffsll(static_cast<long long>(left)) - 1;
              left &= left - 1u;
              ++nb;
            }
          }
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + stage * L::STAGE;
          mbar_arrive_expect_tx(full_bar(stage), static_cast<uint32_t>(nb) * L::SLOT);
#pragma unroll
          for (int j = 0; j < L::G; ++j) {
            if (rg[j] < 0) continue;
            const int r = rg[j];
            const int c = list_c[slot * KM + r];
            const uint32_t sl = st + j * L::SLOT;
            tma_load_3d(sl, &tmX, full_bar(stage), slab * CF, c * S, b);
            tma_load_3d(sl + L::XBOX, &tmX, full_bar(stage), slab * CF + 64, c * S, b);
            if constexpr (!L::PRES) {
#pragma unroll
              for (int ch = 0; ch < L::PCH; ++ch)
                tma_load_3d(sl + L::XB + ch * L::PBOX, &tmP, full_bar(stage), r * S + ch * 64, 0, 0);
            }
          }
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
      for (int s = 0; s < L::STAGES; ++s) {
        if (issued > s) {
          const long long last = ((issued - 1 - s) / L::STAGES) * L::STAGES + s;
          cwait_drain(full_bar(s), static_cast<uint32_t>((last / L::STAGES) & 1));
        }
      }
      if constexpr (L::PRES) cwait_drain(pready_bar, 0);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(CF, S) | (1u << 15);       // A is MN-major
      const uint32_t idesc_res = idesc_bf16_f32(CF, 64) | (1u << 15);  // residual, 64 tokens
      int stage = 0, grp = 0;
      uint32_t phase = 0, grp_phase = 0;
      bool ok = true;
      int it = 0;
      if constexpr (L::PRES) ok = mbar_wait(pready_bar, 0, abort_flag);
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x, ++it) {
        const int slot = it & 1;
        if (!mbar_wait(lfull_bar(slot), (it >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        uint64_t left = 0;  // blocks present
#pragma unroll
        for (int r = 0; r < KM; ++r) left |= (list_c[slot * KM + r] >= 0 ? 1ull : 0ull) << r;
        mbar_arrive(lempty_bar(slot));
#pragma unroll 1
        while (left != 0u) {
          int rg[L::G];  // the group: the producer's pairing of the same present blocks
#pragma unroll
          for (int j = 0; j < L::G; ++j) {
            rg[j] = -1;
            if (left != 0u) {
              rg[j] = __ffsll(static_cast<long long>(left)) - 1;
              left &= left - 1u;
            }
          }
          if (!mbar_wait(tempty_bar(grp), grp_phase ^ 1u, abort_flag) ||
              !mbar_wait(full_bar(stage), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + stage * L::STAGE;
#pragma unroll
          for (int j = 0; j < L::G; ++j) {
            if (rg[j] < 0) continue;
            const int r = rg[j];
            const uint32_t sl = st + j * L::SLOT;
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>((grp * L::G + j) * S);
            // 16 tokens j a step: +2048 bytes (two 8-token atoms) along X's
            // MN-major rows; +32 bytes along P_r's K-major rows, P box every 64 j
#pragma unroll
            for (int kk = 0; kk < S / 16; ++kk) {
              const uint32_t pb = L::PRES ? pbase + r * L::PBOX : sl + L::XB + (kk >> 2) * L::PBOX;
              tc_mma_bf16(d_tmem, cdesc_mn(sl + 2048u * kk, L::XBOX), cdesc_k(pb + 32u * (kk & 3)),
                          idesc, kk != 0);
            }
            if (r == 0) {  // + X_t^T: the residual, one 64-token half at a time
#pragma unroll
              for (int hh = 0; hh < S / 64; ++hh)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  tc_mma_bf16(d_tmem + 64u * hh, cdesc_mn(sl + 8192u * hh + 2048u * kk, L::XBOX),
                              cdesc_k(ibase + 32u * kk), idesc_res, 1u);
            }
          }
          tc_commit(empty_bar(stage));
          tc_commit(tfull_bar(grp));
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if (++grp == L::NGRP) {
            grp = 0;
            grp_phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      tc_commit(drain_bar);
      cwait_drain(drain_bar, 0);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    constexpr int TOK = L::TOK;
    const int quarter = warp & 3;      // TMEM lanes = features 32*quarter .. +31 of the slab
    const int half = (warp - 2) >> 2;  // TMEM columns = tokens TOK*half .. +TOK-1 of the split
    int grp = 0;
    uint32_t grp_phase = 0;
    bool ok = true;
    int it = 0;
    for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x, ++it) {
      const long long seg = tile / a.nslab;
      const int slab = static_cast<int>(tile - seg * a.nslab);
      const int slot = it & 1;
      if (!mbar_wait(lfull_bar(slot), (it >> 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      uint64_t mask = 0;
#pragma unroll 1
      for (int r = 0; r <= a.k && r < KM; ++r) mask |= (list_c[slot * KM + r] >= 0 ? 1ull : 0ull) << r;
      float o[TOK];
#pragma unroll
      for (int i = 0; i < TOK; ++i) o[i] = 0.f;
      const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
      const uint32_t col = static_cast<uint32_t>(half * TOK) + lane_off;
      uint64_t left = mask;  // present blocks not yet added, taken in the MMA issuer's groups
#pragma unroll 1
      while (left != 0u && ok) {
        const int r1 = __ffsll(static_cast<long long>(left)) - 1;
        left &= left - 1u;
        const float w1 = list_w[slot * KM + r1];
        int r2 = -1;
        float w2 = 0.f;
        if constexpr (L::G == 2) {
          if (left != 0u) {
            r2 = __ffsll(static_cast<long long>(left)) - 1;
            left &= left - 1u;
            w2 = list_w[slot * KM + r2];
          }
        }
        if (!(ok = mbar_wait(tfull_bar(grp), grp_phase, abort_flag))) break;
        tc_fence_after();
        const uint32_t t1 = tmem_base + static_cast<uint32_t>(grp * L::G * S) + col;
        const int g = grp;
        if (++grp == L::NGRP) {
          grp = 0;
          grp_phase ^= 1u;
        }
        if constexpr (L::G == 2) {
          if (r2 >= 0) {
            // both blocks of the group with one wait: the second load's latency
            // overlaps the first's
            float v1[32], v2[32];
            tmem_ld32x2(t1, t1 + S, v1, v2);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty_bar(g));
#pragma unroll
            for (int i = 0; i < TOK; ++i) o[i] = fmaf(w2, v2[i], fmaf(w1, v1[i], o[i]));
            continue;
          }
        }
        float v[TOK];
        if constexpr (TOK == 64) {
          tmem_ld64(t1, v);
        } else {
          tmem_ld32(t1, v);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(g));
#pragma unroll
        for (int i = 0; i < TOK; ++i) o[i] = fmaf(w1, v[i], o[i]);
      }
      // the list slot is no longer read by this warp
      __syncwarp();
      if (lane == 0) mbar_arrive(lempty_bar(slot));
      if (!ok) break;
      // fp32 out and/or the split pair, straight to global memory: per token
      // the warp's 32 lanes write 32 consecutive features
      const int f = slab * CF + quarter * 32 + lane;
      if (f < a.d) {
        const long long row0 = seg * S + half * TOK;
        const long long base_off = row0 * a.d + f;
#pragma unroll
        for (int i = 0; i < TOK; ++i) {
          const float y = o[i];
          const long long off = base_off + static_cast<long long>(i) * a.d;
          if (a.out) a.out[off] = y;
          if (a.out_hi) {
            const bf16 h = __float2bfloat16_rn(y);
            a.out_hi[off] = h;
            a.out_lo[off] = __float2bfloat16_rn(y - __bfloat162float(h));
          }
        }
      }
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
    tmem_dealloc(tmem_base, 512);
  }
}

template <int S, int KM>
avey_status run_compress_tc(const CUtensorMap &mx, const CUtensorMap &mp, const CompArgs &a,
                            int grid, cudaStream_t s) {
  using L = CompLayout<S, KM>;
  auto kern = compress_tc_kernel<S, KM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::SMEM));
  if (e != cudaSuccess) {
    set_detail("compress_tc: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  kern<<<grid, C_THR, L::SMEM, s>>>(mx, mp, a);
  AVEY_CHECK_LAUNCH("compress_tc", s);
  return AVEY_OK;
}

template <int S>
avey_status run_compress_tc_k(int k, const CUtensorMap &mx, const CUtensorMap &mp,
                              const CompArgs &a, int grid, cudaStream_t s) {
  if (k + 1 <= 8) return run_compress_tc<S, 8>(mx, mp, a, grid, s);
  if (k + 1 <= 16) return run_compress_tc<S, 16>(mx, mp, a, grid, s);
  if (k + 1 <= 32) return run_compress_tc<S, 32>(mx, mp, a, grid, s);
  return run_compress_tc<S, 33>(mx, mp, a, grid, s);  // k = 32: the target and 32 candidates
}

}  // namespace

bool compress_tc_supported(int S, int d) { return (S == 64 || S == 128) && d % 8 == 0; }

avey_status launch_compress_tc(const bf16 *x, int B, int N, int d, int S, int k, int t0, int nr,
                               const int32_t *idx, const float *w, const bf16 *P, float *out,
                               bf16 *hi, bf16 *lo, cudaStream_t s) {
  AVEY_REQUIRE(compress_tc_supported(S, d), AVEY_ERR_UNSUPPORTED,
               "compress_tc: S=%d, d=%d unsupported", S, d);
  const int n = (N + S - 1) / S;
  CUtensorMap mx, mp;
  const uint64_t rs = static_cast<uint64_t>(d) * 2;
  if (!encode_map(&mx, false, x, d, N, B, rs, rs * N, 64, S, 128)) return AVEY_ERR_CUDA;
  const uint64_t ps = static_cast<uint64_t>(k + 1) * S * 2;
  if (!encode_map(&mp, false, P, static_cast<uint64_t>(k + 1) * S, S, 1, ps, ps * S, 64, S, 128))
    return AVEY_ERR_CUDA;
  CompArgs a{};
  a.N = N;
  a.d = d;
  a.n = n;
  a.k = k;
  a.nslab = (d + CF - 1) / CF;
  a.t0 = t0;
  a.nr = nr;
  const long long tiles = static_cast<long long>(B) * nr * a.nslab;
  AVEY_REQUIRE(tiles <= 0x7fffffffll, AVEY_ERR_UNSUPPORTED, "compress_tc: too many tiles");
  a.num_tiles = static_cast<int>(tiles);
  a.idx = idx;
  a.w = w;
  a.x = x;
  a.out = out;
  a.out_hi = hi;
  a.out_lo = lo;
  a.status = device_status_word();
  const int grid = std::max(1, std::min(a.num_tiles, sm_count()));
  if (S == 64) return run_compress_tc_k<64>(k, mx, mp, a, grid, s);
  return run_compress_tc_k<128>(k, mx, mp, a, grid, s);
}

}  // namespace avey
