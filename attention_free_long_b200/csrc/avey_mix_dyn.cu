// avey_mix_dyn.cu -- the dynamic contextualizer of a split-size layer on the
// tcgen05 tensor cores (papernotes 关键设计 2-3; paperlayer summary §4.2):
//   G_ij = N(z_i).N(z_j)                       within each split of S tokens
//   Gt_ij = G_ij / (sum_j G_ij + eps)          (eq. 6)
//   c = Gt Z_t
// and, with COUPLED, the original Avey's coupled causal map
//   M_ij = V_ij G_ij for j <= i (0 otherwise),  c = M Z_t   (no row sums).
// Z_t is an activation split pair (hi, lo bf16 planes); c is written as a
// split pair, in place or to a separate buffer.
//
// One persistent, warp-specialised kernel, one CTA per SM.  A tile is 128
// consecutive token rows: 128 / S whole splits (S in {16, 32, 64, 128}).
//   1. Gram.  The tile's hi rows stream through a ring of TMA stages (128
//      rows x 64 features, K-major, 128-byte swizzle); each stage is both
//      operands of four 128 x 128 x 16 MMAs, so TMEM holds R = Z_hi Z_hi^T of
//      the whole tile (the blocks outside the diagonal splits go unused).
//   2. eq. 6 in the epilogue warps, two threads per TMEM lane (token row i),
//      each on half of the row's split: 1/|z_i| = 1/sqrt(R_ii) from the
//      diagonal, the cosines R_ij / (|z_i| |z_j|), the row sum (two halves
//      met in shared memory) and Gt = cos / (sum + eps) in fp32, split to a
//      bf16 pair and written into shared memory as the K-major A operand of
//      step 3 (block-diagonal: the zeros outside the splits are written once).
//   3. Apply.  Z_t is read straight from the token-major activation as an
//      MN-major B operand: TMA boxes of 64 features x 64 tokens per plane.
//      Per 16 tokens three MMAs (Gt_hi Z_hi + Gt_lo Z_hi + Gt_hi Z_lo) into
//      one of two 64-column accumulators; the epilogue (32 columns per warp)
//      splits c to a pair, stages it in a 4 KB swizzled buffer per warp and
//      stores it by TMA (a thread holds a row, so direct stores would touch 32
//      rows per instruction: measured 1.5x slower), which leaves room for
//      seven ring stages (112 KB of loads in flight).
// The hi rows are read twice (steps 1 and 3); the second read is close
// enough in time to the first to be served mostly from L2.  A tile's Gram is
// loaded and summed while the CTA's previous tile is applied (its chunks
// interleaved with the apply stages in the ring), so a tile waits only for
// eq. 6 between its Gram and its apply.
// Roles: warp 0 TMA producer, warp 1 TMEM allocation and MMA issue, warps 2-9
// epilogue (two per TMEM lane quarter).  Every wait is bounded
// (avey_common.cuh); a wait that runs out records AVEY_ERR_DEVICE_TIMEOUT and
// the kernel drains and returns.
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

constexpr int DT = 128;                    // token rows per tile
constexpr int DF = 64;                     // features per Gram chunk and per apply tile
constexpr int D_EPI = 8;                   // epilogue warps: two per TMEM lane quarter
constexpr int D_THR = 64 + 32 * D_EPI;
constexpr uint32_t D_STAGE = 16384;        // 128 rows x 64 features, or 2 planes x 64 x 64
constexpr uint32_t D_ZBOX = 8192;          // one plane of an apply stage: 64 tokens x 64 features
constexpr int D_STAGES = 7;
constexpr uint32_t D_GT_CHUNK = 16384;     // 128 rows x 64 tokens of one Gt plane
constexpr uint32_t D_GT_PLANE = 2 * D_GT_CHUNK;
constexpr uint32_t D_OUT = 2048;           // one plane of a warp's output box: 32 rows x 32
constexpr uint32_t D_GT_OFF = D_STAGES * D_STAGE;
constexpr uint32_t D_OUT_OFF = D_GT_OFF + 2 * D_GT_PLANE;
constexpr uint32_t D_CTRL_OFF = D_OUT_OFF + D_EPI * 2 * D_OUT;
constexpr uint32_t D_CTRL = 4096;  // barriers, TMEM address, flag, 1/norms [2][128], sums [2][2][128]
constexpr uint32_t D_SMEM = D_CTRL_OFF + D_CTRL + 1024;  // + alignment slack
static_assert(D_SMEM <= 232448, "shared memory budget");
static_assert(D_GT_OFF % 1024 == 0 && D_OUT_OFF % 1024 == 0 && D_CTRL_OFF % 1024 == 0,
              "swizzled buffers need 1024-byte alignment");
constexpr uint32_t D_COLS = 256;           // TMEM: Gram [0, 128), accumulators 128 + 64 a

struct DynArgs {
  int rows;       // T = blocks * S
  int mt;         // mixed features
  int nk;         // ceil(mt / 64)
  int num_tiles;  // ceil(T / 128)
  float eps;
  const bf16 *V;  // COUPLED: [S, S]
  int *status;
};

// K-major operand, 128-byte swizzle: 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t dyn_desc_k(uint32_t a) {
  return static_cast<uint64_t>((a >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1u) << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
         (static_cast<uint64_t>(2u) << 61);
}
// MN-major operand of 64 MN elements, 128-byte swizzle: one 128-byte row per
// K index, 8-row atoms 1024 bytes apart along K.
__device__ __forceinline__ uint64_t dyn_desc_mn(uint32_t a) {
  return static_cast<uint64_t>((a >> 4) & 0x3FFFu) | (static_cast<uint64_t>(D_ZBOX >> 4) << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
         (static_cast<uint64_t>(2u) << 61);
}

__device__ __forceinline__ void dyn_drain_wait(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// Gram chunks of the next tile to have issued after the apply pair jn of the
// current one (nk pairs, nk chunks): none in the first half, then two per
// pair, all by the last.
__host__ __device__ constexpr int gram_chunks_after(int jn, int nk) {
  return 2 * (jn + 1) - nk < 0 ? 0 : (2 * (jn + 1) - nk > nk ? nk : 2 * (jn + 1) - nk);
}

// Byte offset of element (row, k) of a K-major tile with 128-byte rows and
// 128-byte swizzle (16-byte chunk c of row r sits at chunk c ^ (r % 8)).
__device__ __forceinline__ uint32_t sw128_off(int row, int k) {
  return static_cast<uint32_t>((row >> 3) * 1024 + (row & 7) * 128 +
                               ((((k >> 3) ^ row) & 7) << 4) + (k & 7) * 2);
}

// Contextualizer kinds of the kernel: eq. 6, the coupled causal map, or the
// static map V (shared by every split; no Gram).
enum { MIX_DYNAMIC = 0, MIX_COUPLED = 1, MIX_STATIC = 2 };

template <int S, int KIND>
__global__ void __launch_bounds__(D_THR, 1)
    split_mix_tc_kernel(const __grid_constant__ CUtensorMap tmG,
                      const __grid_constant__ CUtensorMap tmZh,
                      const __grid_constant__ CUtensorMap tmZl,
                      const __grid_constant__ CUtensorMap tmOh,
                      const __grid_constant__ CUtensorMap tmOl, const DynArgs a) {
  static_assert(S == 16 || S == 32 || S == 64 || S == 128, "split size");
  constexpr bool kGram = KIND != MIX_STATIC;     // eq. 6 / coupled: Gram per tile
  constexpr bool kCoupled = KIND == MIX_COUPLED;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t *base = smem_raw + pad;
  const uint32_t sbase = raw_s + pad;
  const uint32_t gth = sbase + D_GT_OFF, gtl = gth + D_GT_PLANE;
  uint8_t *ctrl = base + D_CTRL_OFF;
  const uint32_t cbase = sbase + D_CTRL_OFF;
  // control block: full[s] @8s, empty[s] @128+8s (s < 16), tfull[2] @256,
  // tempty[2] @272, gfull @288, gempty @296, gtready @304, gtfree @312,
  // drain @320, tmem base @328, abort flag @332, 1/norms [2][128] fp32 @512,
  // half-row sums [2][2][128] fp32 @1536
  static_assert(D_STAGES <= 16, "control block holds at most 16 stages");
  auto full_bar = [&](int s) { return cbase + 8u * s; };
  auto empty_bar = [&](int s) { return cbase + 128u + 8u * s; };
  auto tfull_bar = [&](int i) { return cbase + 256u + 8u * i; };
  auto tempty_bar = [&](int i) { return cbase + 272u + 8u * i; };
  const uint32_t gfull_bar = cbase + 288u, gempty_bar = cbase + 296u;
  const uint32_t gtready_bar = cbase + 304u, gtfree_bar = cbase + 312u;
  const uint32_t drain_bar = cbase + 320u;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(ctrl + 328);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 332);
  float *s_rn = reinterpret_cast<float *>(ctrl + 512);
  float *s_rs = reinterpret_cast<float *>(ctrl + 1536);
  static_assert(1536 + 4 * 128 * 4 <= D_CTRL, "control block size");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < D_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), D_EPI);
    }
    mbar_init(gfull_bar, 1);
    mbar_init(gempty_bar, D_EPI);
    mbar_init(gtready_bar, D_EPI);
    mbar_init(gtfree_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(ctrl + 328), D_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmG);
    prefetch_tmap(&tmZh);
    prefetch_tmap(&tmZl);
    prefetch_tmap(&tmOh);
    prefetch_tmap(&tmOl);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      auto next = [&]() -> bool {
        if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) return false;
        mbar_arrive_expect_tx(full_bar(stage), D_STAGE);
        return true;
      };
      auto advance = [&]() {
        ++issued;
        if (++stage == D_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      };
      // Stage order (the MMA issuer consumes the same): the first tile's Gram
      // chunks, then for every tile its apply stages, two per 64 features,
      // with the Gram chunks of the CTA's next tile placed after the pairs of
      // the second half (gram_chunks_after), so that the next Gram is loaded
      // and summed while this tile is applied.
      auto gram_chunk = [&](int r0, int kc) -> bool {
        if (!next()) return false;
        tma_load_3d(sbase + stage * D_STAGE, &tmG, full_bar(stage), kc * DF, r0, 0);
        advance();
        return true;
      };
      if (kGram && static_cast<int>(blockIdx.x) < a.num_tiles)
        for (int kc = 0; kc < a.nk && ok; ++kc) ok = gram_chunk(blockIdx.x * DT, kc);
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        const int r0 = tile * DT;
        const int tn = tile + static_cast<int>(gridDim.x);  // this CTA's next tile
        int g = 0;                                           // its Gram chunks issued
        for (int jn = 0; jn < a.nk && ok; ++jn) {  // apply: 64 features x 64 tokens x 2 planes
          for (int kh = 0; kh < 2; ++kh) {
            if (!(ok = next())) break;
            const uint32_t st = sbase + stage * D_STAGE;
            tma_load_3d(st, &tmZh, full_bar(stage), jn * DF, r0 + kh * 64, 0);
            tma_load_3d(st + D_ZBOX, &tmZl, full_bar(stage), jn * DF, r0 + kh * 64, 0);
            advance();
          }
          // the next Gram's chunks ride along the second half of this apply,
          // two per 64 features, so that their second read (the next apply)
          // follows soon enough to come from L2
          if (kGram && tn < a.num_tiles)
            for (; ok && g < gram_chunks_after(jn, a.nk); ++g) ok = gram_chunk(tn * DT, g);
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      // wait (bounded) for the loads still in flight before the CTA exits
      for (int s = 0; s < D_STAGES; ++s) {
        if (issued > s) {
          const long long last = ((issued - 1 - s) / D_STAGES) * D_STAGES + s;
          dyn_drain_wait(full_bar(s), static_cast<uint32_t>((last / D_STAGES) & 1));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t id_gram = idesc_bf16_f32(DT, DT);
      const uint32_t id_apply = idesc_bf16_f32(DT, DF) | (1u << 16);  // B is MN-major
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0, gphase = 0;  // gphase: parity of the tile being applied
      bool ok = true;
      // one 64-feature chunk of a tile's Gram into TMEM columns [0, 128)
      auto gram_chunk = [&](int kc) -> bool {
        if (!mbar_wait(full_bar(stage), phase, abort_flag)) return false;
        tc_fence_after();
        const uint32_t st = sbase + stage * D_STAGE;
#pragma unroll
        for (int kk = 0; kk < DF / 16; ++kk) {
          const uint64_t d = dyn_desc_k(st + 32u * kk);
          tc_mma_bf16(tmem_base, d, d, id_gram, (kc | kk) != 0);
        }
        tc_commit(empty_bar(stage));
        if (++stage == D_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
        return true;
      };
      if (kGram && static_cast<int>(blockIdx.x) < a.num_tiles) {
        // the first tile's Gram (later tiles' Grams ride along the apply)
        ok = mbar_wait(gempty_bar, 1u, abort_flag);
        if (ok) tc_fence_after();
        for (int kc = 0; kc < a.nk && ok; ++kc) ok = gram_chunk(kc);
        if (ok) tc_commit(gfull_bar);
      }
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        const bool next_gram = kGram && tile + static_cast<int>(gridDim.x) < a.num_tiles;
        int g = 0;  // the next tile's Gram chunks issued
        // c = Gt Z_t (or V Z_t), 64 features at a time; the static V is
        // written once, before the first tile
        if (kGram || tile == static_cast<int>(blockIdx.x)) {
          if (!(ok = mbar_wait(gtready_bar, kGram ? gphase : 0u, abort_flag))) break;
          tc_fence_after();
        }
        for (int jn = 0; jn < a.nk && ok; ++jn) {
          if (!(ok = mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag))) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + 128u + static_cast<uint32_t>(acc * DF);
          for (int kh = 0; kh < 2; ++kh) {
            if (!(ok = mbar_wait(full_bar(stage), phase, abort_flag))) break;
            tc_fence_after();
            const uint32_t st = sbase + stage * D_STAGE;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // 16 tokens: +32 bytes along Gt's K-major rows, +2048 bytes (two
              // 8-token atoms) along Z's MN-major rows
              const uint64_t ah = dyn_desc_k(gth + kh * D_GT_CHUNK + 32u * kk);
              const uint64_t al = dyn_desc_k(gtl + kh * D_GT_CHUNK + 32u * kk);
              const uint64_t bh = dyn_desc_mn(st + 2048u * kk);
              const uint64_t bl = dyn_desc_mn(st + D_ZBOX + 2048u * kk);
              tc_mma_bf16(d_tmem, ah, bh, id_apply, (kh | kk) != 0);
              if constexpr (kGram) tc_mma_bf16(d_tmem, al, bh, id_apply, 1u);  // V is exact in bf16
              tc_mma_bf16(d_tmem, ah, bl, id_apply, 1u);
            }
            tc_commit(empty_bar(stage));
            if (++stage == D_STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          tc_commit(tfull_bar(acc));
          acc ^= 1;
          if (acc == 0) acc_phase ^= 1u;
          if (next_gram) {
            // the next tile's Gram chunks: its TMEM was released when this
            // tile's eq. 6 read the Gram (before gtready), so this wait passes
            const int upto = gram_chunks_after(jn, a.nk);
            if (g == 0 && upto > 0) {
              if (!(ok = mbar_wait(gempty_bar, gphase, abort_flag))) break;
              tc_fence_after();
            }
            for (; ok && g < upto; ++g) ok = gram_chunk(g);
            if (!ok) break;
          }
        }
        if (!ok) break;
        if (next_gram) tc_commit(gfull_bar);
        tc_commit(gtfree_bar);  // the tile's MMAs no longer read Gt
        gphase ^= 1u;
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      tc_commit(drain_bar);
      dyn_drain_wait(drain_bar, 0);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    // Eight warps, two per TMEM lane quarter: warp (quarter, h) owns token row
    // `row` and half h of the work on it (half of the row's split in eq. 6,
    // 32 of each 64-feature accumulator in the apply).
    const int quarter = warp & 3;          // TMEM lanes 32 quarter .. + 31
    const int h = (warp - 2) >> 2;
    const int row = quarter * 32 + lane;   // token row within the tile
    constexpr int NQ = S / 2;              // split columns per thread
    constexpr int LW = NQ >= 32 ? NQ : 32; // Gram columns a warp loads
    const int srow = row / S * S;          // first row of this row's split
    const int q0 = srow + h * NQ;          // first split column of this thread
    // warp-uniform load column: this half of the split for S >= 64, else the
    // warp's own 32 columns (S = 32: its split; S = 16: its two splits)
    const int lcol = S >= 64 ? q0 : quarter * 32;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    uint8_t *ob = base + D_OUT_OFF + (warp - 2) * 2 * D_OUT;  // staging: hi, lo
    const uint32_t ob_s = sbase + D_OUT_OFF + (warp - 2) * 2 * D_OUT;
    // Gt outside the diagonal splits stays zero: clear this row of both planes
    // once (half h clears K chunk h)
    {
      const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int pl = 0; pl < 2; ++pl)
#pragma unroll
        for (int c = 0; c < 8; ++c)
          *reinterpret_cast<uint4 *>(base + D_GT_OFF + pl * D_GT_PLANE + h * D_GT_CHUNK +
                                     sw128_off(row, c * 8)) = z;
    }
    if constexpr (!kGram) {
      // the static map: V in every diagonal S x S block of the hi plane, once
      // (after every row's zeros: the two threads of a row cleared different
      // K chunks, and this thread's V columns may lie in the other's)
      named_bar_sync(1, 32 * D_EPI);
#pragma unroll
      for (int q = 0; q < NQ; q += 8) {
        const uint4 vv = *reinterpret_cast<const uint4 *>(a.V + (row - srow) * S + h * NQ + q);
        const int k = q0 + q;
        *reinterpret_cast<uint4 *>(base + D_GT_OFF + (k / 64) * D_GT_CHUNK + sw128_off(row, k % 64)) = vv;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(gtready_bar);
    }
    int acc = 0;
    uint32_t acc_phase = 0, gphase = 0;
    bool ok = true;
    // Every epilogue warp runs the same number of named barriers (two per
    // tile): after a failed wait a warp stops waiting and working but still
    // walks the tile loop, so the others never wait for it.
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      const int r0 = tile * DT;
      if constexpr (kGram) {
      float *rn = s_rn + (gphase & 1u) * 128;
      float *rs = s_rs + (gphase & 1u) * 256;
      // ---- eq. 6 from the Gram ----
      float g[NQ];
      const bool got = ok && mbar_wait(gfull_bar, gphase, abort_flag);
      if (got) {
        tc_fence_after();
        float v[LW];
#pragma unroll
        for (int q = 0; q < LW; q += 32)
          tmem_ld32(tmem_base + lane_off + static_cast<uint32_t>(lcol + q),
                    *reinterpret_cast<float(*)[32]>(&v[q]));
        // this thread's NQ split columns, at offset q0 - lcol in v
        const int off = q0 - lcol;  // 0 for S >= 64; 0 or 16 (S = 32); 0, 8, 16, 24 (S = 16)
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          if constexpr (S >= 64) {
            g[q] = v[q];
          } else if constexpr (S == 32) {
            g[q] = off ? v[16 + q] : v[q];
          } else {
            g[q] = off == 0 ? v[q] : off == 8 ? v[8 + q] : off == 16 ? v[16 + q] : v[24 + q];
          }
        }
        // the diagonal R_ii sits in exactly one of the row's two threads
        if (row >= q0 && row < q0 + NQ) {
          float gii = 0.f;
#pragma unroll
          for (int q = 0; q < NQ; ++q)
            if (q0 + q == row) gii = g[q];
          rn[row] = 1.0f / fmaxf(sqrtf(gii), 1e-12f);
        }
      } else {
        ok = false;
      }
      tc_fence_before();
      __syncwarp();
      if (got && lane == 0) mbar_arrive(gempty_bar);  // the Gram's TMEM may be overwritten
      named_bar_sync(1, 32 * D_EPI);                   // every row's 1/|z| is in place
      float part = 0.f;
      if (ok) {
        const float ri = rn[row];
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          g[q] = g[q] * (ri * rn[q0 + q]);  // the cosine
          part += g[q];
        }
      }
      rs[h * 128 + row] = part;
      named_bar_sync(1, 32 * D_EPI);                   // both halves of every row sum
      gphase ^= 1u;
      if (!ok) continue;
      if constexpr (kCoupled) {
        const int i = row - srow;
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          const int j = h * NQ + q;
          g[q] = j <= i ? __bfloat162float(a.V[i * S + j]) * g[q] : 0.f;
        }
      } else {
        const float dinv = 1.0f / (rs[row] + rs[128 + row] + a.eps);
#pragma unroll
        for (int q = 0; q < NQ; ++q) g[q] = g[q] * dinv;
      }
      // the previous tile's MMAs must be done with Gt before it is rewritten
      // (gphase now has the parity of the previous tile)
      if (!(ok = mbar_wait(gtfree_bar, gphase, abort_flag))) continue;
#pragma unroll
      for (int q = 0; q < NQ; q += 8) {
        uint4 hv, lv;
        split_pack(g[q], g[q + 1], hv.x, lv.x);
        split_pack(g[q + 2], g[q + 3], hv.y, lv.y);
        split_pack(g[q + 4], g[q + 5], hv.z, lv.z);
        split_pack(g[q + 6], g[q + 7], hv.w, lv.w);
        const int k = q0 + q;  // token column of Gt
        const uint32_t o = (k / 64) * D_GT_CHUNK + sw128_off(row, k % 64);
        *reinterpret_cast<uint4 *>(base + D_GT_OFF + o) = hv;
        *reinterpret_cast<uint4 *>(base + D_GT_OFF + D_GT_PLANE + o) = lv;
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(gtready_bar);
      } else if (!ok) {
        continue;
      }
      // ---- c tiles: TMEM -> split pair -> swizzled staging -> TMA store ----
      for (int jn = 0; jn < a.nk; ++jn) {
        if (!(ok = mbar_wait(tfull_bar(acc), acc_phase, abort_flag))) break;
        tc_fence_after();
        float c[32];
        tmem_ld32(tmem_base + lane_off + 128u + static_cast<uint32_t>(acc * DF + h * 32), c);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        const int x0 = jn * DF + h * 32;
        // rows past T and features past m_t are never stored
        if (r0 + quarter * 32 >= a.rows || x0 >= a.mt) continue;
        // the warp's previous store has finished reading the staging buffer
        if (lane == 0) bulk_wait_read<0>();
        __syncwarp();
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
          uint32_t hv[4], lv[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) split_pack(c[8 * gq + 2 * u], c[8 * gq + 2 * u + 1], hv[u], lv[u]);
          const uint32_t o = static_cast<uint32_t>(lane * 64 + ((gq ^ ((lane >> 1) & 3)) << 4));
          *reinterpret_cast<uint4 *>(ob + o) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
          *reinterpret_cast<uint4 *>(ob + D_OUT + o) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_3d(&tmOh, ob_s, x0, r0 + quarter * 32, 0);
          tma_store_3d(&tmOl, ob_s + D_OUT, x0, r0 + quarter * 32, 0);
          bulk_commit();
        }
      }
    }
    if (!ok) {
      *abort_flag = 1;
      record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
    }
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, D_COLS);
  }
}

template <int S, int KIND>
avey_status run_split_mix_tc(const CUtensorMap *maps, const DynArgs &args, cudaStream_t s) {
  auto kern = split_mix_tc_kernel<S, KIND>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(D_SMEM));
  if (e != cudaSuccess) {
    set_detail("split mix: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  const int grid = std::min(args.num_tiles, sm_count());
  kern<<<grid, D_THR, D_SMEM, s>>>(maps[0], maps[1], maps[2], maps[3], maps[4], args);
  AVEY_CHECK_LAUNCH(KIND == MIX_DYNAMIC ? "dynamic_mix_tc" : KIND == MIX_COUPLED ? "coupled_mix_tc"
                                                                                : "static_mix_tc",
                    s);
  return AVEY_OK;
}

template <int KIND>
avey_status run_split_mix_s(int S, const CUtensorMap *maps, const DynArgs &args, cudaStream_t s) {
  switch (S) {
    case 16: return run_split_mix_tc<16, KIND>(maps, args, s);
    case 32: return run_split_mix_tc<32, KIND>(maps, args, s);
    case 64: return run_split_mix_tc<64, KIND>(maps, args, s);
    default: return run_split_mix_tc<128, KIND>(maps, args, s);
  }
}

avey_status split_mix_tc(int kind, const bf16 *zt, int64_t ld_zt, int64_t plane_zt, bf16 *out,
                         int64_t ld_out, int64_t plane_out, int blocks, int S, int mt, float eps,
                         const bf16 *V, cudaStream_t s) {
  AVEY_REQUIRE(S == 16 || S == 32 || S == 64 || S == 128, AVEY_ERR_UNSUPPORTED,
               "split mix: S=%d unsupported (16, 32, 64 or 128)", S);
  AVEY_REQUIRE(mt >= 8 && mt % 8 == 0 && ld_zt % 8 == 0 && ld_out % 8 == 0 && aligned16(zt) &&
                   aligned16(out) && aligned16(zt + plane_zt) && aligned16(out + plane_out) &&
                   (V == nullptr || aligned16(V)),
               AVEY_ERR_INVALID_ARG,
               "split mix: mt, ld multiples of 8 and 16-byte aligned planes and V required");
  AVEY_REQUIRE(kind == MIX_DYNAMIC || V != nullptr, AVEY_ERR_INVALID_ARG, "split mix: V is required");
  if (blocks <= 0) return AVEY_OK;
  const long long T = static_cast<long long>(blocks) * S;
  AVEY_REQUIRE(T <= 0x7fffff00ll, AVEY_ERR_UNSUPPORTED, "split mix: too many rows");
  CUtensorMap maps[5];
  const uint64_t zrow = static_cast<uint64_t>(ld_zt) * 2, orow = static_cast<uint64_t>(ld_out) * 2;
  if (!encode_bf16_map(&maps[0], zt, mt, T, 1, zrow, zrow * T, DT)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&maps[1], zt, mt, T, 1, zrow, zrow * T, 64)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&maps[2], zt + plane_zt, mt, T, 1, zrow, zrow * T, 64)) return AVEY_ERR_CUDA;
  // c leaves in boxes of 32 features x 32 rows, 64-byte swizzle
  if (!encode_map(&maps[3], false, out, mt, T, 1, orow, orow * T, 32, 32, 64)) return AVEY_ERR_CUDA;
  if (!encode_map(&maps[4], false, out + plane_out, mt, T, 1, orow, orow * T, 32, 32, 64))
    return AVEY_ERR_CUDA;
  DynArgs args{};
  args.rows = static_cast<int>(T);
  args.mt = mt;
  args.nk = (mt + DF - 1) / DF;
  args.num_tiles = static_cast<int>((T + DT - 1) / DT);
  args.eps = eps;
  args.V = V;
  args.status = device_status_word();
  if (kind == MIX_DYNAMIC) return run_split_mix_s<MIX_DYNAMIC>(S, maps, args, s);
  if (kind == MIX_COUPLED) return run_split_mix_s<MIX_COUPLED>(S, maps, args, s);
  return run_split_mix_s<MIX_STATIC>(S, maps, args, s);
}

}  // namespace

avey_status launch_dynamic_mix_x2(const bf16 *zt, int64_t ld_zt, int64_t plane_zt, bf16 *out,
                                  int64_t ld_out, int64_t plane_out, int blocks, int S, int mt,
                                  float eps, cudaStream_t s) {
  return split_mix_tc(MIX_DYNAMIC, zt, ld_zt, plane_zt, out, ld_out, plane_out, blocks, S, mt, eps,
                      nullptr, s);
}

avey_status launch_coupled_mix_x2(const bf16 *V, const bf16 *zt, int64_t ld_zt, int64_t plane_zt,
                                  bf16 *out, int64_t ld_out, int64_t plane_out, int blocks, int S,
                                  int mt, cudaStream_t s) {
  return split_mix_tc(MIX_COUPLED, zt, ld_zt, plane_zt, out, ld_out, plane_out, blocks, S, mt, 0.f,
                      V, s);
}

avey_status launch_static_mix_x2(const bf16 *V, const bf16 *zt, int64_t ld, int blocks, int S,
                                 int mt, int64_t plane, bf16 *out, int64_t ld_out,
                                 int64_t plane_out, cudaStream_t s) {
  return split_mix_tc(MIX_STATIC, zt, ld, plane, out, ld_out, plane_out, blocks, S, mt, 0.f, V, s);
}

}  // namespace avey
