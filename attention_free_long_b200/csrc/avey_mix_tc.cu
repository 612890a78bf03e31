// avey_mix_tc.cu -- the contextualizer over long token blocks (256 or 512
// tokens) on the tcgen05 tensor cores, for the processor without neural
// compression (Avey-B paperlayer summary §4.3; papernotes 关键设计 2-3):
//   c_b = A_b Z_b,   A_b = V (static, shared by every block) or the block's
//                    Gt pair (dynamic, from avey_mix_long.cu's Gram kernels)
// for every block b of SL tokens, Z_b the block's tail activations as a bf16
// split pair.
//
// One persistent, warp-specialised kernel; a tile is (block, 128 rows i,
// 256 features f), accumulated in TMEM over the SL tokens j:
//   * two stages of 64 tokens (stages of 32 tokens with 64-byte-swizzled A
//     boxes allowed four or five stages but measured slower);
//   * A (rows i, K = j) is K-major: a TMA box of 64 tokens x 128 rows, 128-byte
//     swizzle, as in the other tcgen05 kernels;
//   * B = Z_b (N = f, K = j) is read straight from the token-major activation:
//     it is MN-major, four TMA boxes of 64 features x 64 tokens per plane, so
//     that each token row of 64 features is one 128-byte swizzled row, eight
//     token rows form a 1024-byte atom (the descriptor's stride offset), and
//     the four 64-feature groups sit 8 KB apart (its leading offset);
//   * MMAs per 16 tokens: A Z_hi and A Z_lo, plus A_lo Z_hi for the Gt pair;
//   * the epilogue writes c as a split pair to a separate buffer (the tiles of
//     other row blocks still read Z_b), which the fuser then reads in place of
//     Z's tail.
// Roles: warp 0 TMA producer, warp 1 TMEM allocation and MMA issue, warps 2-5
// epilogue (one per TMEM lane quarter).  Two accumulators of 256 columns let
// the epilogue of one tile overlap the MMAs of the next.  Every wait is
// bounded (avey_common.cuh).
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

constexpr int MT = 128, NT = 256, KT = 64;  // tile rows, tile features, tokens per stage
constexpr int kEpiW = 4, kThr = 64 + 32 * kEpiW;
constexpr uint32_t kCols = 512;
constexpr uint32_t A_BOX = MT * KT * 2;     // 16 KB: 128 rows x 64 tokens
constexpr uint32_t Z_BOX = 64 * KT * 2;     // 8 KB: 64 features x 64 tokens
constexpr uint32_t Z_PLANE = 4 * Z_BOX;     // 256 features

template <int A_PLANES>
struct MixLayout {
  static constexpr uint32_t STAGE = A_PLANES * A_BOX + 2 * Z_PLANE;
  static constexpr int STAGES = 2;
  static constexpr uint32_t TILES = STAGES * STAGE;
  static constexpr uint32_t CTRL = 1024;
  static constexpr uint32_t SMEM = TILES + CTRL + 1024;
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct MixArgs {
  int SL, mt, blocks;
  int iblocks, fblocks, num_tiles;
  int a_batched;  // A's TMA z coordinate is the block (Gt) or 0 (V)
  bf16 *chi, *clo;
  long long ldc;
  int *status;
};

// K-major operand, 128-byte swizzle: 8-row atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_k(uint32_t a) {
  return static_cast<uint64_t>((a >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1u) << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
         (static_cast<uint64_t>(2u) << 61);
}
// MN-major operand, 128-byte swizzle: 64 contiguous MN elements per 128-byte
// row (one row per K index), 8-row atoms 1024 bytes apart along K (stride
// offset), 64-element MN groups Z_BOX bytes apart (leading offset).
__device__ __forceinline__ uint64_t desc_mn(uint32_t a) {
  return static_cast<uint64_t>((a >> 4) & 0x3FFFu) | (static_cast<uint64_t>(Z_BOX >> 4) << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
         (static_cast<uint64_t>(2u) << 61);
}

__device__ __forceinline__ void mix_decode(const MixArgs &a, int tile, int &b, int &ib, int &fb) {
  fb = tile % a.fblocks;
  const int r = tile / a.fblocks;
  ib = r % a.iblocks;
  b = r / a.iblocks;
}

__device__ __forceinline__ void wait_drain_mix(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

template <int A_PLANES>
__global__ void __launch_bounds__(kThr, 1)
    mix_tc_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                  const __grid_constant__ CUtensorMap tmZ0, const __grid_constant__ CUtensorMap tmZ1,
                  const MixArgs a) {
  using L = MixLayout<A_PLANES>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t *ctrl = smem_raw + pad + L::TILES;
  const uint32_t sbase = raw_s + pad;
  const uint32_t cbase = sbase + L::TILES;
  // control block (room for up to 8 stages): full[s] @8s, empty[s] @64+8s,
  // tfull[2] @128, tempty[2] @144, drain @160, tmem base @168, abort flag @172
  static_assert(L::STAGES <= 8, "control block holds at most 8 stages");
  auto full_bar = [&](int s) { return cbase + 8u * s; };
  auto empty_bar = [&](int s) { return cbase + 64u + 8u * s; };
  auto tfull_bar = [&](int i) { return cbase + 128u + 8u * i; };
  auto tempty_bar = [&](int i) { return cbase + 144u + 8u * i; };
  const uint32_t drain_bar = cbase + 160u;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(ctrl + 168);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 172);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < L::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), kEpiW);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(ctrl + 168), kCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmA0);
    if (A_PLANES == 2) prefetch_tmap(&tmA1);
    prefetch_tmap(&tmZ0);
    prefetch_tmap(&tmZ1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int kchunks = a.SL / KT;

  if (warp == 0) {
    // -------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        int b, ib, fb;
        mix_decode(a, tile, b, ib, fb);
        const int az = a.a_batched ? b : 0;
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + stage * L::STAGE;
          mbar_arrive_expect_tx(full_bar(stage), L::STAGE);
          tma_load_3d(st, &tmA0, full_bar(stage), kc * KT, ib * MT, az);
          if (A_PLANES == 2) tma_load_3d(st + A_BOX, &tmA1, full_bar(stage), kc * KT, ib * MT, az);
          const uint32_t zb = st + A_PLANES * A_BOX;
          const int zrow = b * a.SL + kc * KT;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tma_load_3d(zb + q * Z_BOX, &tmZ0, full_bar(stage), fb * NT + q * 64, zrow, 0);
            tma_load_3d(zb + Z_PLANE + q * Z_BOX, &tmZ1, full_bar(stage), fb * NT + q * 64, zrow, 0);
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
          wait_drain_mix(full_bar(s), static_cast<uint32_t>((last / L::STAGES) & 1));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(MT, NT) | (1u << 16);  // B is MN-major
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NT);
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + stage * L::STAGE;
          const uint32_t zb = st + A_PLANES * A_BOX;
#pragma unroll
          for (int kk = 0; kk < KT / 16; ++kk) {
            // 16 tokens: +32 bytes along A's K-major rows, +2048 bytes (two
            // 8-token atoms) along Z's MN-major rows
            const uint64_t dah = desc_k(st + 32u * kk);
            const uint64_t dzh = desc_mn(zb + 2048u * kk);
            const uint64_t dzl = desc_mn(zb + Z_PLANE + 2048u * kk);
            tc_mma_bf16(d_tmem, dah, dzh, idesc, (kc | kk) != 0);
            tc_mma_bf16(d_tmem, dah, dzl, idesc, 1u);
            if (A_PLANES == 2) tc_mma_bf16(d_tmem, desc_k(st + A_BOX + 32u * kk), dzh, idesc, 1u);
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
      wait_drain_mix(drain_bar, 0);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;  // TMEM lanes 32*quarter .. +31
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      int b, ib, fb;
      mix_decode(a, tile, b, ib, fb);
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + static_cast<uint32_t>(acc * NT) + (static_cast<uint32_t>(quarter * 32) << 16);
      const long long row = static_cast<long long>(b) * a.SL + ib * MT + quarter * 32 + lane;
      bf16 *ch = a.chi + row * a.ldc;
      bf16 *cl = a.clo + row * a.ldc;
#pragma unroll 1
      for (int c0 = 0; c0 < NT; c0 += 64) {
        float v[64];
        tmem_ld64(taddr + c0, v);
        const int f0 = fb * NT + c0;
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          if (f0 + 8 * g >= a.mt) break;
          uint4 h, l;
          split_pack(v[8 * g], v[8 * g + 1], h.x, l.x);
          split_pack(v[8 * g + 2], v[8 * g + 3], h.y, l.y);
          split_pack(v[8 * g + 4], v[8 * g + 5], h.z, l.z);
          split_pack(v[8 * g + 6], v[8 * g + 7], h.w, l.w);
          *reinterpret_cast<uint4 *>(ch + f0 + 8 * g) = h;
          *reinterpret_cast<uint4 *>(cl + f0 + 8 * g) = l;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
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
    tmem_dealloc(tmem_base, kCols);
  }
}

// ---- Gt of the dynamic mix over long blocks: the hi-plane Gram on tcgen05 ----
//   Gt_ij = (z_i . z_j) inv_n[i] inv_n[j] inv_d[i]
// (inv_n = 1/|z| of the hi rows, inv_d = 1/(row sum + eps), both from
// long_dyn_prep).  A tile is (block, 128 rows i, 256 columns j); both operands
// are the block's hi rows, K-major (features contiguous), in 64-feature
// chunks: A boxes of 128 rows, B boxes of 256 rows.
constexpr uint32_t G_A = 128 * 64 * 2, G_B = 256 * 64 * 2;  // 16 KB, 32 KB
constexpr uint32_t G_STAGE = G_A + G_B;
constexpr int G_STAGES = 4;
constexpr uint32_t G_SMEM = G_STAGES * G_STAGE + 1024 + 1024;
static_assert(G_SMEM <= 232448, "shared memory budget");

struct GramArgs {
  int SL, mt, blocks, iblocks, jblocks, num_tiles;
  const float *inv_n, *inv_d;
  bf16 *gt;
  long long gt_plane;
  int *status;
};

__global__ void __launch_bounds__(kThr, 1)
    gram_tc_kernel(const __grid_constant__ CUtensorMap tmZa, const __grid_constant__ CUtensorMap tmZb,
                   const GramArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t *ctrl = smem_raw + pad + G_STAGES * G_STAGE;
  const uint32_t sbase = raw_s + pad;
  const uint32_t cbase = sbase + G_STAGES * G_STAGE;
  static_assert(G_STAGES <= 4, "the Gram control block holds at most 4 stages");
  // control block: full[4] @0, empty[4] @32, tfull[2] @64, tempty[2] @80,
  // drain @96, tmem base @104, abort flag @108
  auto full_bar = [&](int s) { return cbase + 8u * s; };
  auto empty_bar = [&](int s) { return cbase + 32u + 8u * s; };
  auto tfull_bar = [&](int i) { return cbase + 64u + 8u * i; };
  auto tempty_bar = [&](int i) { return cbase + 80u + 8u * i; };
  const uint32_t drain_bar = cbase + 96u;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(ctrl + 104);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 108);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < G_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), kEpiW);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(ctrl + 104), kCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmZa);
    prefetch_tmap(&tmZb);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  const int kchunks = (a.mt + 63) / 64;
  auto decode = [&](int tile, int &b, int &ib, int &jb) {
    jb = tile % a.jblocks;
    const int r = tile / a.jblocks;
    ib = r % a.iblocks;
    b = r / a.iblocks;
  };

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        int b, ib, jb;
        decode(tile, b, ib, jb);
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + stage * G_STAGE;
          mbar_arrive_expect_tx(full_bar(stage), G_STAGE);
          tma_load_3d(st, &tmZa, full_bar(stage), kc * 64, b * a.SL + ib * 128, 0);
          tma_load_3d(st + G_A, &tmZb, full_bar(stage), kc * 64, b * a.SL + jb * 256, 0);
          ++issued;
          if (++stage == G_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      for (int s = 0; s < G_STAGES; ++s) {
        if (issued > s) {
          const long long last = ((issued - 1 - s) / G_STAGES) * G_STAGES + s;
          wait_drain_mix(full_bar(s), static_cast<uint32_t>((last / G_STAGES) & 1));
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, 256);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 256);
        for (int kc = 0; kc < kchunks; ++kc) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + stage * G_STAGE;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_bf16(d_tmem, desc_k(st + 32u * kk), desc_k(st + G_A + 32u * kk), idesc,
                        (kc | kk) != 0);
          tc_commit(empty_bar(stage));
          if (++stage == G_STAGES) {
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
      wait_drain_mix(drain_bar, 0);
    }
  } else {
    const int quarter = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.num_tiles; tile += gridDim.x) {
      int b, ib, jb;
      decode(tile, b, ib, jb);
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t taddr =
          tmem_base + static_cast<uint32_t>(acc * 256) + (static_cast<uint32_t>(quarter * 32) << 16);
      const int i = ib * 128 + quarter * 32 + lane;
      const long long rb = static_cast<long long>(b) * a.SL;
      const float ri = __ldg(a.inv_n + rb + i) * __ldg(a.inv_d + rb + i);
      const float *nj = a.inv_n + rb + jb * 256;
      bf16 *gh = a.gt + (rb + i) * a.SL + jb * 256;
      bf16 *gl = gh + a.gt_plane;
#pragma unroll 1
      for (int c0 = 0; c0 < 256; c0 += 64) {
        float v[64];
        tmem_ld64(taddr + c0, v);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float4 n0 = __ldg(reinterpret_cast<const float4 *>(nj + c0 + 8 * g));
          const float4 n1 = __ldg(reinterpret_cast<const float4 *>(nj + c0 + 8 * g + 4));
          uint4 h, l;
          split_pack(v[8 * g] * ri * n0.x, v[8 * g + 1] * ri * n0.y, h.x, l.x);
          split_pack(v[8 * g + 2] * ri * n0.z, v[8 * g + 3] * ri * n0.w, h.y, l.y);
          split_pack(v[8 * g + 4] * ri * n1.x, v[8 * g + 5] * ri * n1.y, h.z, l.z);
          split_pack(v[8 * g + 6] * ri * n1.z, v[8 * g + 7] * ri * n1.w, h.w, l.w);
          *reinterpret_cast<uint4 *>(gh + c0 + 8 * g) = h;
          *reinterpret_cast<uint4 *>(gl + c0 + 8 * g) = l;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty_bar(acc));
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
    tmem_dealloc(tmem_base, kCols);
  }
}

template <int A_PLANES>
avey_status run_mix_tc(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &z0,
                       const CUtensorMap &z1, const MixArgs &args, cudaStream_t s) {
  using L = MixLayout<A_PLANES>;
  auto kern = mix_tc_kernel<A_PLANES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(L::SMEM));
  if (e != cudaSuccess) {
    set_detail("mix_tc: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  const int grid = std::min(args.num_tiles, sm_count());
  kern<<<grid, kThr, L::SMEM, s>>>(a0, a1, z0, z1, args);
  AVEY_CHECK_LAUNCH("mix_tc", s);
  return AVEY_OK;
}

}  // namespace

avey_status launch_long_mix_tc(const bf16 *a_hi, const bf16 *a_lo, bool a_batched, const bf16 *zhi,
                               const bf16 *zlo, int64_t ldz, int blocks, int SL, int mt, bf16 *chi,
                               bf16 *clo, cudaStream_t s) {
  AVEY_REQUIRE(SL == 256 || SL == 512, AVEY_ERR_UNSUPPORTED,
               "long mix: block of %d tokens unsupported (256 or 512)", SL);
  AVEY_REQUIRE(mt >= 8 && mt % 8 == 0 && ldz % 8 == 0, AVEY_ERR_INVALID_ARG,
               "long mix: mt and ld must be multiples of 8");
  AVEY_REQUIRE(aligned16(a_hi) && (!a_lo || aligned16(a_lo)) && aligned16(zhi) && aligned16(zlo) &&
                   aligned16(chi) && aligned16(clo),
               AVEY_ERR_INVALID_ARG, "long mix: pointers must be 16-byte aligned");
  const long long T = static_cast<long long>(blocks) * SL;
  CUtensorMap ma0, ma1, mz0, mz1;
  const uint64_t arow = static_cast<uint64_t>(SL) * 2, ablk = arow * SL;
  if (!encode_bf16_map(&ma0, a_hi, SL, SL, a_batched ? blocks : 1, arow, ablk, MT)) return AVEY_ERR_CUDA;
  if (a_lo && !encode_bf16_map(&ma1, a_lo, SL, SL, a_batched ? blocks : 1, arow, ablk, MT))
    return AVEY_ERR_CUDA;
  const uint64_t zrow = static_cast<uint64_t>(ldz) * 2;
  if (!encode_bf16_map(&mz0, zhi, mt, T, 1, zrow, zrow * T, KT)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&mz1, zlo, mt, T, 1, zrow, zrow * T, KT)) return AVEY_ERR_CUDA;
  MixArgs args{};
  args.SL = SL;
  args.mt = mt;
  args.blocks = blocks;
  args.iblocks = SL / MT;
  args.fblocks = (mt + NT - 1) / NT;
  const long long tiles = static_cast<long long>(blocks) * args.iblocks * args.fblocks;
  AVEY_REQUIRE(tiles <= 0x7fffffffll, AVEY_ERR_UNSUPPORTED, "long mix: too many tiles");
  args.num_tiles = static_cast<int>(tiles);
  args.a_batched = a_batched ? 1 : 0;
  args.chi = chi;
  args.clo = clo;
  args.ldc = mt;
  args.status = device_status_word();
  if (a_lo) return run_mix_tc<2>(ma0, ma1, mz0, mz1, args, s);
  return run_mix_tc<1>(ma0, ma0, mz0, mz1, args, s);
}

avey_status launch_long_gram_tc(const bf16 *zhi, int64_t ldz, int blocks, int SL, int mt,
                                const float *inv_n, const float *inv_d, bf16 *gt, cudaStream_t s) {
  AVEY_REQUIRE(SL == 256 || SL == 512, AVEY_ERR_UNSUPPORTED,
               "long Gram: block of %d tokens unsupported (256 or 512)", SL);
  AVEY_REQUIRE(mt >= 8 && mt % 8 == 0 && ldz % 8 == 0 && aligned16(zhi) && aligned16(gt),
               AVEY_ERR_INVALID_ARG, "long Gram: mt, ld multiples of 8; 16-byte aligned pointers");
  const long long T = static_cast<long long>(blocks) * SL;
  const uint64_t zrow = static_cast<uint64_t>(ldz) * 2;
  CUtensorMap za, zb;
  if (!encode_bf16_map(&za, zhi, mt, T, 1, zrow, zrow * T, 128)) return AVEY_ERR_CUDA;
  if (!encode_bf16_map(&zb, zhi, mt, T, 1, zrow, zrow * T, 256)) return AVEY_ERR_CUDA;
  GramArgs g{};
  g.SL = SL;
  g.mt = mt;
  g.blocks = blocks;
  g.iblocks = SL / 128;
  g.jblocks = SL / 256;
  const long long tiles = static_cast<long long>(blocks) * g.iblocks * g.jblocks;
  AVEY_REQUIRE(tiles <= 0x7fffffffll, AVEY_ERR_UNSUPPORTED, "long Gram: too many tiles");
  g.num_tiles = static_cast<int>(tiles);
  g.inv_n = inv_n;
  g.inv_d = inv_d;
  g.gt = gt;
  g.gt_plane = static_cast<long long>(blocks) * SL * SL;
  g.status = device_status_word();
  cudaError_t e = cudaFuncSetAttribute(gram_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(G_SMEM));
  if (e != cudaSuccess) {
    set_detail("gram_tc: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  const int grid = std::min(g.num_tiles, sm_count());
  gram_tc_kernel<<<grid, kThr, G_SMEM, s>>>(za, zb, g);
  AVEY_CHECK_LAUNCH("gram_tc", s);
  return AVEY_OK;
}

}  // namespace avey
