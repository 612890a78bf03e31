// avey_maxsim2.cu -- MaxSim split scores on CTA pairs (tcgen05 cta_group::2),
// the ranker's dominant step for S in {32, 64, 128} (Avey-B paperlayer summary
// §3 and papernotes 整体框架: score(t, c) = sum over the rows of split t of the
// max cosine to a row of split c).  The cosines are formed from the raw bf16
// dot products and the scales 1/|x_i|, 1/|x_j|; only the [B, n, n] split
// scores reach HBM.  Laid out for two SMs per tile:
//
//   * A cluster of two CTAs owns a 256 x 256 tile of G = X X^T: each CTA
//     holds 128 of its rows in TMEM (fp32), loads those 128 rows of X (A) and
//     one half (128 rows) of the column tile (B) with TMA; CTA 0 issues
//     tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16), which reads A and
//     both halves of B across the pair.  Per FLOP each SM moves a third fewer
//     bytes from L2 than with 128 x 256 tiles on one SM.
//   * Tiles are square in 256-row blocks, so the triangular order is simply
//     nt >= mt: the diagonal tile yields the scores of its own splits from
//     row maxima; a tile right of the diagonal yields score(t -> c) from row
//     maxima and score(c -> t) from column maxima over each target split's
//     rows (a target split never straddles the two CTAs).
//   * Roles per CTA (320 threads): warp 0 TMA producer; warp 1 TMEM
//     allocation (both CTAs) and the MMA issue (CTA 0); warps 2-9 epilogue,
//     two per TMEM lane quarter, one per 128-column half.
//   * Barriers: each CTA's loads complete on CTA 0's "full" barrier; the MMA
//     commit frees the stage in both CTAs and publishes the accumulator to
//     both; both CTAs' epilogue warps release the accumulator to CTA 0.
//     Every wait is bounded (avey_common.cuh); every load fills only the
//     issuing CTA's own shared memory.
//   * Tiles are visited in groups of 32 row blocks (the group's rows stay in
//     L2 while its column blocks stream past); a launch may compute only the
//     tiles t with t % nparts == part (one long sequence across GPUs).
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

constexpr int PT = 256;                       // tile edge (rows and columns)
constexpr int BK = 64;                        // K chunk (128-byte swizzled rows)
constexpr int kStages = 6;
constexpr int kEpi = 8;
constexpr int kThreads = 64 + 32 * kEpi;
constexpr uint32_t kTmemCols = 512;           // two 128 x 256 fp32 accumulators per CTA
constexpr int kGroup = 32;                    // 256-row tiles per L2 group
constexpr int kRedCands = 16;
constexpr uint32_t HALF_BYTES = 128 * BK * 2;  // 16 KB: 128 rows x 64 bf16
constexpr uint32_t STAGE_BYTES = 2 * HALF_BYTES;
constexpr uint32_t TILES_BYTES = kStages * STAGE_BYTES;
constexpr uint32_t CTRL_BYTES = 14336;
constexpr uint32_t SMEM_BYTES = TILES_BYTES + CTRL_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

struct PairArgs {
  int n;              // splits per sequence
  int tiles;          // 256-blocks per sequence (rows = columns)
  long long slots;    // triangular-order slots per sequence
  int num_tiles;      // B * slots
  int part, nparts;   // this launch computes the tiles t with t % nparts == part
  int kchunks;
  float *scores;      // [B, n, n]
  const float *inv_norm;
  int rs_ld;
  int *status;
};

__device__ __forceinline__ long long pair_prefix(long long g, long long tn) {
  return kGroup * g * tn - static_cast<long long>(kGroup) * kGroup * g * (g - 1) / 2;
}

// Slots of group g: its row blocks (32, fewer in the last group) times the
// column blocks 32g .. tiles-1.
__device__ __forceinline__ int group_slots(int tiles, int g, int &rows) {
  rows = min(kGroup, tiles - g * kGroup);
  return rows * (tiles - g * kGroup);
}

// One pair's walk over the slots first, first + step, ... of the triangular
// order.  Group g holds row blocks 32g .. 32g+31 and column blocks
// 32g .. tiles-1, row block fastest; slots left of the diagonal (nt < mt)
// hold no work and every role skips them alike.  Only the first slot is
// located from scratch (a square root); each step then moves the in-group
// offset on and crosses whole groups and sequences, a few integer operations
// per tile on the MMA issuer's critical path.
struct PairCursor {
  long long tile;  // global slot (sequence-major)
  int b, g;        // sequence, group
  int x;           // slot inside group g
  int size, rows;  // slots and row blocks of group g
};

__device__ __forceinline__ void cursor_init(const PairArgs &a, PairCursor &c, long long first) {
  c.tile = first;
  c.b = static_cast<int>(first / a.slots);
  const long long x = first - static_cast<long long>(c.b) * a.slots;
  const long long tn = a.tiles;
  const double A = static_cast<double>(kGroup) * tn + kGroup * kGroup / 2.0;
  const double disc = A * A - 2.0 * kGroup * kGroup * static_cast<double>(x);
  long long g = static_cast<long long>((A - sqrt(disc > 0 ? disc : 0)) / (kGroup * kGroup));
  if (g < 0) g = 0;
  while (g > 0 && pair_prefix(g, tn) > x) --g;
  while (pair_prefix(g + 1, tn) <= x && (g + 1) * kGroup < a.tiles) ++g;
  c.g = static_cast<int>(g);
  c.x = static_cast<int>(x - pair_prefix(g, tn));
  c.size = group_slots(a.tiles, c.g, c.rows);
}

__device__ __forceinline__ void cursor_next(const PairArgs &a, PairCursor &c, int step) {
  c.tile += step;
  if (c.tile >= a.num_tiles) return;
  c.x += step;
  while (c.x >= c.size) {
    c.x -= c.size;
    if (++c.g * kGroup >= a.tiles) {
      c.g = 0;
      ++c.b;
    }
    c.size = group_slots(a.tiles, c.g, c.rows);
  }
}

// (row block, column block) of the cursor's slot; false left of the diagonal.
__device__ __forceinline__ bool cursor_tile(const PairCursor &c, int &mt, int &nt) {
  const int q = c.rows == kGroup ? (c.x >> 5) : c.x / c.rows;
  nt = c.g * kGroup + q;
  mt = c.g * kGroup + (c.x - q * c.rows);
  return nt >= mt;
}

__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// One epilogue warp: its 32 rows (TMEM lanes) x its 128 columns, whose
// scales c_j sit in the warp's shared-memory copy cs.  With
// v = x_i . x_j, r_i = 1/|x_i| and c_j = 1/|x_j| (both >= 0), the cosine's
// row maximum is r_i * max_j (v c_j) and its column maximum c_j * max_i (v r_i);
// each direction takes one packed product per two entries.  Row maxima per
// candidate split, summed over the warp's rows -> red; column maxima of v r_i
// over the warp's rows -> cm (only right of the diagonal; c_j is applied when
// they are summed).
template <int S>
__device__ __forceinline__ void pair_rows(uint32_t taddr, int lane, int quarter, int half, float *red,
                                          float *cm, const float *cs, float row_scale,
                                          bool need_col) {
  constexpr int CH_PER_CAND = S / 32;
  const float2 r2 = make_float2(row_scale, row_scale);
  float m = -INFINITY;
#pragma unroll 1
  for (int pr = 0; pr < 2; ++pr) {
    const int ch0 = 4 * half + 2 * pr;  // 32-column chunk index inside the 256-column tile
    const float4 *cs4 = reinterpret_cast<const float4 *>(cs + 2 * pr * 32);
    float v[64];
    tmem_ld64(taddr + ch0 * 32, v);
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int ch = ch0 + u;
      float p[32];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const float4 c = cs4[8 * u + q];  // the same address in every lane: a broadcast
        const float2 a = fmul2(make_float2(v[32 * u + 4 * q], v[32 * u + 4 * q + 1]), make_float2(c.x, c.y));
        const float2 b = fmul2(make_float2(v[32 * u + 4 * q + 2], v[32 * u + 4 * q + 3]), make_float2(c.z, c.w));
        p[4 * q] = a.x;
        p[4 * q + 1] = a.y;
        p[4 * q + 2] = b.x;
        p[4 * q + 3] = b.y;
      }
      if (ch % CH_PER_CAND == 0) m = -INFINITY;
      m = fmaxf(m, max32(p));
      if (ch % CH_PER_CAND == CH_PER_CAND - 1) {
        float t = m * row_scale;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
        if (lane == 0) red[quarter * kRedCands + ch / CH_PER_CAND] = t;
      }
      if (need_col) {
        // column maxima of v r_i over this warp's 32 rows: one warp reduction per column
        float4 *dst = reinterpret_cast<float4 *>(cm + (quarter * 8 + ch) * 32);
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const float2 a = fmul2(make_float2(v[32 * u + 4 * g], v[32 * u + 4 * g + 1]), r2);
          const float2 b = fmul2(make_float2(v[32 * u + 4 * g + 2], v[32 * u + 4 * g + 3]), r2);
          const float4 mx = make_float4(warp_max(a.x), warp_max(a.y), warp_max(b.x), warp_max(b.y));
          if (lane == 0) dst[g] = mx;
        }
      }
    }
  }
}

// Leader warp of one half: scores of this CTA's target splits against the
// half's candidate splits (row maxima), and, right of the diagonal, of the
// half's splits as targets against this CTA's splits (column maxima times
// 1/|x_j| from the warp's copy cs, summed over the candidate's columns).
template <int S>
__device__ __forceinline__ void pair_write(const PairArgs &a, const float *red, const float *cm,
                                           const float *cs, int lane, int b,
                                           int t0, int c0, int half, bool need_col) {
  constexpr int TS = 128 / S, PER = S / 32, CB = 128 / S;
  float *scores = a.scores + static_cast<long long>(b) * a.n * a.n;
  for (int e = lane; e < TS * CB; e += 32) {
    const int ts = e / CB, cl = e - (e / CB) * CB;
    float sc = 0.f;
#pragma unroll
    for (int q = 0; q < PER; ++q) sc += red[(ts * PER + q) * kRedCands + half * CB + cl];
    const int t = t0 + ts, c = c0 + cl;
    if (t < a.n && c < a.n) scores[static_cast<long long>(t) * a.n + c] = sc;
  }
  if (!need_col) return;
  for (int ts = 0; ts < TS; ++ts) {
    for (int cl = 0; cl < CB; ++cl) {
      float sum = 0.f;
#pragma unroll
      for (int u = 0; u < PER; ++u) {
        const int ch = half * 4 + cl * PER + u;
        float mx = cm[((ts * PER) * 8 + ch) * 32 + lane];
#pragma unroll
        for (int q = 1; q < PER; ++q) mx = fmaxf(mx, cm[((ts * PER + q) * 8 + ch) * 32 + lane]);
        sum += mx * cs[(cl * PER + u) * 32 + lane];
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      const int t = t0 + ts, c = c0 + cl;
      if (lane == 0 && t < a.n && c < a.n) scores[static_cast<long long>(c) * a.n + t] = sum;
    }
  }
}

template <int S>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    maxsim_pair_kernel(const __grid_constant__ CUtensorMap tmX, const PairArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t *ctrl = smem_raw + pad + TILES_BYTES;
  const uint32_t sbase = raw_s + pad;
  const uint32_t cbase = sbase + TILES_BYTES;
  static_assert(kStages <= 8, "the control block holds at most 8 stages");
  // control block: full[6] @0, empty[6] @64, tfull[2] @128, tempty[2] @144,
  // redbar[4] @160, redfree[4] @192, drain @224, tmem base @232, abort @236,
  // red @256, column maxima @2048, column scales [8 epilogue warps][128] @10240
  auto full_bar = [&](int s) { return cbase + 8u * s; };
  auto empty_bar = [&](int s) { return cbase + 64u + 8u * s; };
  auto tfull_bar = [&](int i) { return cbase + 128u + 8u * i; };
  auto tempty_bar = [&](int i) { return cbase + 144u + 8u * i; };
  auto red_bar = [&](int i) { return cbase + 160u + 8u * i; };
  auto red_free = [&](int i) { return cbase + 192u + 8u * i; };
  const uint32_t drain_bar = cbase + 224u;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(ctrl + 232);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 236);
  float *red = reinterpret_cast<float *>(ctrl + 256);
  float *cmx = reinterpret_cast<float *>(ctrl + 2048);
  float *csx = reinterpret_cast<float *>(ctrl + 10240);
  static_assert(10240 + 8 * 128 * 4 <= CTRL_BYTES, "control block size");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int first = pair * a.nparts + a.part, step = npairs * a.nparts;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 2 * kEpi);  // both CTAs' epilogue warps (used in CTA 0)
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(red_bar(i), 4);
      mbar_init(red_free(i), 1);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) prefetch_tmap(&tmX);
  cluster_sync_all();  // barriers of both CTAs initialised before any remote use
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(ctrl + 232), kTmemCols);
    tmem_relinquish_pair();
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
      PairCursor cur;
      cursor_init(a, cur, first);
      for (; cur.tile < a.num_tiles && ok; cursor_next(a, cur, step)) {
        int mt, nt;
        if (!cursor_tile(cur, mt, nt)) continue;
        const int b = cur.b;
        for (int kc = 0; kc < a.kchunks; ++kc) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * STAGE_BYTES);
          const uint32_t full0 = mapa_shared(full_bar(stage), 0);
          const uint32_t st = sbase + stage * STAGE_BYTES;
          tma_load_3d_pair(st, &tmX, full0, kc * BK, mt * PT + rank * 128, b);
          tma_load_3d_pair(st + HALF_BYTES, &tmX, full0, kc * BK, nt * PT + rank * 128, b);
          ++issued;
          if (++stage == kStages) {
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
      for (int s = 0; s < kStages; ++s) {
        if (issued > s) {
          const long long last = ((issued - 1 - s) / kStages) * kStages + s;
          wait_drain(empty_bar(s), static_cast<uint32_t>((last / kStages) & 1));
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------- MMA issue (CTA 0)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * 128, PT);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      PairCursor cur;
      cursor_init(a, cur, first);
      for (; cur.tile < a.num_tiles && ok; cursor_next(a, cur, step)) {
        int mt, nt;
        if (!cursor_tile(cur, mt, nt)) continue;
        if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * PT);
        for (int kc = 0; kc < a.kchunks; ++kc) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + stage * STAGE_BYTES;
          const uint64_t da = sdesc_k_sw128(st);
          const uint64_t db = sdesc_k_sw128(st + HALF_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_bf16_pair(d_tmem, da + 2u * kk, db + 2u * kk, idesc, (kc | kk) != 0);
          tc_commit_pair_both(empty_bar(stage));
          if (++stage == kStages) {
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
      wait_drain(drain_bar, 0);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t tempty_r0 = mapa_shared(tempty_bar(0), 0), tempty_r1 = mapa_shared(tempty_bar(1), 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    PairCursor cur;
    cursor_init(a, cur, first);
    for (; cur.tile < a.num_tiles; cursor_next(a, cur, step)) {
      int mt, nt;
      if (!cursor_tile(cur, mt, nt)) continue;
      const int b = cur.b;
      const int row0 = mt * PT + static_cast<int>(rank) * 128;  // this CTA's rows of the tile
      const float *rs = a.inv_norm + static_cast<long long>(b) * a.rs_ld;
      // the scales of this warp's rows and of its half's 128 columns, loaded
      // before the accumulator wait so that their latency hides behind it
      const float row_scale = rs[row0 + quarter * 32 + lane];
      const float4 col4 = __ldg(reinterpret_cast<const float4 *>(rs + nt * PT + half * 128) + lane);
      if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
      float *cs = csx + (warp - 2) * 128;  // read by this warp alone, after this store
      reinterpret_cast<float4 *>(cs)[lane] = col4;
      __syncwarp();
      const int rb = acc * 2 + half;
      if (!mbar_wait(red_free(rb), acc_phase ^ 1u, abort_flag)) {
        ok = false;
        break;
      }
      const uint32_t taddr =
          tmem_base + static_cast<uint32_t>(acc * PT) + (static_cast<uint32_t>(quarter * 32) << 16);
      const bool need_col = nt > mt;
      float *red_acc = red + acc * 8 * kRedCands;
      float *cm_acc = cmx + acc * (4 * 8 * 32);
      pair_rows<S>(taddr, lane, quarter, half, red_acc, cm_acc, cs, row_scale, need_col);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_cluster(acc ? tempty_r1 : tempty_r0);  // release this accumulator to the MMA issuer
        mbar_arrive(red_bar(rb));
      }
      if (warp == 2 + 4 * half) {
        if (!mbar_wait(red_bar(rb), acc_phase, abort_flag)) {
          ok = false;
        } else {
          pair_write<S>(a, red_acc, cm_acc, cs, lane, b, row0 / S,
                        (nt * PT + half * 128) / S, half, need_col);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(red_free(rb));
      }
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
  // Both CTAs past their loops: the pair's MMAs have drained (CTA 0 waited on
  // the drain commit) and no remote arrival is still on its way.
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
  cluster_sync_all();
}

template <int S>
avey_status run_pair(const CUtensorMap &mx, PairArgs a, cudaStream_t st) {
  auto kern = maxsim_pair_kernel<S>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(SMEM_BYTES));
  if (e != cudaSuccess) {
    set_detail("maxsim_pair: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
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
    cfg.dynamicSmemBytes = SMEM_BYTES;
    int clusters = 0;
    e = cudaOccupancyMaxActiveClusters(&clusters, kern, &cfg);
    if (e != cudaSuccess || clusters < 1) {
      set_detail("maxsim_pair: no resident CTA pair (%s)", cudaGetErrorString(e));
      return AVEY_ERR_CUDA;
    }
    cap = std::min(clusters, sm_count() / 2);
  }
  const int mine = (a.num_tiles - a.part + a.nparts - 1) / a.nparts;  // tiles of this part
  const int pairs = std::max(1, std::min(mine, cap));
  kern<<<2 * pairs, kThreads, SMEM_BYTES, st>>>(mx, a);
  AVEY_CHECK_LAUNCH("maxsim_pair", st);
  return AVEY_OK;
}

}  // namespace

avey_status launch_maxsim_pair(const bf16 *x, const float *inv_norm, int B, int N, int R, int rs_ld,
                               int d, int S, int n, float *scores, cudaStream_t s, int part,
                               int nparts) {
  CUtensorMap mx;
  const uint64_t rs = static_cast<uint64_t>(d) * 2, bs = rs * static_cast<uint64_t>(N);
  if (!encode_bf16_map(&mx, x, d, N, B, rs, bs, 128)) return AVEY_ERR_CUDA;
  PairArgs a{};
  a.n = n;
  a.tiles = (R + PT - 1) / PT;
  long long slots = 0;
  for (long long g = 0; g * kGroup < a.tiles; ++g)
    slots += std::min<long long>(kGroup, a.tiles - g * kGroup) * (a.tiles - g * kGroup);
  a.slots = slots;
  if (slots * B > 0x7fffffffll || rs_ld < a.tiles * PT) {
    set_detail("maxsim_pair: problem too large");
    return AVEY_ERR_UNSUPPORTED;
  }
  a.num_tiles = static_cast<int>(slots * B);
  a.part = part;
  a.nparts = nparts;
  a.kchunks = (d + BK - 1) / BK;
  a.scores = scores;
  a.inv_norm = inv_norm;
  a.rs_ld = rs_ld;
  a.status = device_status_word();
  switch (S) {
    case 32: return run_pair<32>(mx, a, s);
    case 64: return run_pair<64>(mx, a, s);
    case 128: return run_pair<128>(mx, a, s);
    default: set_detail("maxsim_pair: S=%d unsupported", S); return AVEY_ERR_UNSUPPORTED;
  }
}

}  // namespace avey
