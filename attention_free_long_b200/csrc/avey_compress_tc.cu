// avey_compress_tc.cu -- neural compression with residual on tcgen05, S = 64
// (papernotes 关键设计 4, eq. 8; paperlayer summary §4.3, App. H):
//   out(t) = sum_{r=0..k} w_r P_r X_{c_r} + X_t,   c_0 = t, w_0 = 1.
//
// A tile is (target split t, 128-feature slab); per retrieved block r the
// tensor cores compute the transposed partial product
//   D_r[f, i] = sum_j X_{c_r}[j, f] P[i, rS + j]     (M = 128 f, N = 64 i, K = 64 j)
// with the block's 64 token rows gathered by TMA straight from the token-major
// embeddings (an MN-major A operand: boxes of 64 features x 64 tokens, 128-byte
// swizzle) and P_r as the K-major B operand.  Every D_r lands in its own TMEM
// buffer; the epilogue (thread = feature f) adds w_r D_r into fp32 registers,
// so the weight multiplies the fp32 product and the bf16 inputs are never
// re-rounded; block 0 also accumulates X_t^T I (the residual, exact), and the
// epilogue writes fp32 plus the split pair (per token, the warp's 32 lanes
// store 32 consecutive features).
// The kernel is bound by HBM: (k+1) gathered 64 x d bf16 blocks in, 64 x d x 8
// bytes out per split; eight stages of 24 KB keep 192 KB of loads in flight.
// Roles: warp 0 TMA producer, warp 1 TMEM allocation and MMA issue, warps 2-9
// epilogue (two per TMEM lane quarter = 32 features, each on 32 of the
// split's 64 tokens).  Every wait is bounded.
#include <algorithm>

#include "avey_common.cuh"
#include "avey_internal.h"

namespace avey {
namespace {

constexpr int CS = 64;                        // split size handled here
constexpr int CF = 128;                       // features per tile (M)
constexpr int C_EPI = 8, C_THR = 64 + 32 * C_EPI;
constexpr int C_TOK = CS / 2;                 // tokens per epilogue warp
constexpr uint32_t C_XBOX = 64 * CS * 2;      // 8 KB: 64 features x 64 tokens
constexpr uint32_t C_PBOX = CS * CS * 2;      // 8 KB: P_r, 64 i x 64 j
constexpr uint32_t C_STAGE = 2 * C_XBOX + C_PBOX;
constexpr int C_STAGES = 6;
constexpr int C_NACC = 8;                     // TMEM buffers of 64 columns
constexpr uint32_t C_IDENT = CS * CS * 2;     // 8 KB: the 64 x 64 identity (B operand)
constexpr uint32_t C_W32 = C_TOK * 32 * 4;    // 4 KB: one warp's fp32 output [32 i][32 f]
constexpr uint32_t C_W16 = C_TOK * 32 * 2;    // 2 KB: one bf16 plane of it
constexpr uint32_t C_WSTG = C_W32 + 2 * C_W16;
constexpr uint32_t C_SMEM = C_STAGES * C_STAGE + C_IDENT + C_EPI * C_WSTG + 1024 + 1024;
static_assert(C_SMEM <= 232448, "shared memory budget");

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
// token), 8-token atoms 1024 bytes apart, the two 64-feature groups C_XBOX apart.
__device__ __forceinline__ uint64_t cdesc_mn(uint32_t a) {
  return static_cast<uint64_t>((a >> 4) & 0x3FFFu) | (static_cast<uint64_t>(C_XBOX >> 4) << 16) |
         (static_cast<uint64_t>(1024u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
         (static_cast<uint64_t>(2u) << 61);
}

__device__ __forceinline__ void cwait_drain(uint32_t bar, uint32_t parity) {
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (globaltimer_ns() - t0 > kWaitLimitNs) return;
  }
}

// The block list of target t (local row seg = b*nr + t - t0 of idx / w), all
// loads issued at once: split c[r] and weight wr[r] of block r <= k, c = -1
// for no block (every role skips it alike; out-of-range indices are recorded
// by the producer and skipped).  KM >= k + 1 keeps the list in registers.
template <int KM>
__device__ __forceinline__ void block_list(const CompArgs &a, long long seg, int t, bool record,
                                           int (&c)[KM], float (&wr)[KM]) {
  c[0] = t;
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
#pragma unroll
  for (int r = 1; r < KM; ++r) {
    if (c[r] < -1 || c[r] >= a.n) {
      if (record) record_status(a.status, AVEY_ERR_DEVICE_BOUNDS);
      c[r] = -1;
    }
  }
}

template <int KM>
__global__ void __launch_bounds__(C_THR, 1)
    compress_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmP,
                       const __grid_constant__ CUtensorMap tmO, const __grid_constant__ CUtensorMap tmOh,
                       const __grid_constant__ CUtensorMap tmOl, const CompArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t *ident = smem_raw + pad + C_STAGES * C_STAGE;
  uint8_t *ostage = ident + C_IDENT;  // per epilogue warp: fp32 [64][32], hi, lo
  uint8_t *ctrl = ostage + C_EPI * C_WSTG;
  const uint32_t sbase = raw_s + pad;
  const uint32_t ibase = sbase + C_STAGES * C_STAGE;
  const uint32_t obase = ibase + C_IDENT;
  const uint32_t cbase = obase + C_EPI * C_WSTG;
  static_assert(C_STAGES <= 8 && C_NACC <= 8, "the control block holds at most 8 of each");
  // control block: full[8] @0, empty[8] @64, tfull[8] @128, tempty[8] @192,
  // drain @256, tmem base @264, abort flag @268
  auto full_bar = [&](int s) { return cbase + 8u * s; };
  auto empty_bar = [&](int s) { return cbase + 64u + 8u * s; };
  auto tfull_bar = [&](int i) { return cbase + 128u + 8u * i; };
  auto tempty_bar = [&](int i) { return cbase + 192u + 8u * i; };
  const uint32_t drain_bar = cbase + 256u;
  volatile uint32_t *tmem_holder = reinterpret_cast<volatile uint32_t *>(ctrl + 264);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(ctrl + 268);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C_STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < C_NACC; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), C_EPI);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(ctrl + 264), 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmP);
    prefetch_tmap(&tmO);
  }
  // The residual X_t enters block 0's accumulator through the tensor cores:
  // D_0 += X_t^T I with I the 64 x 64 identity, a K-major B operand in the
  // 128-byte-swizzled layout (row i = 64 bf16; its 16-byte chunk q sits at
  // chunk q ^ (i & 7)).  Products with 1 and 0 are exact, so D_0 gains X_t
  // exactly, in fp32.
  for (int e = threadIdx.x; e < static_cast<int>(C_IDENT / 16); e += C_THR)
    reinterpret_cast<uint4 *>(ident)[e] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  if (threadIdx.x < CS) {
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
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        const long long seg = tile / a.nslab;  // b * nr + (t - t0)
        const int slab = static_cast<int>(tile - seg * a.nslab);
        const int b = static_cast<int>(seg / a.nr);
        const int t = a.t0 + static_cast<int>(seg - static_cast<long long>(b) * a.nr);
        int cl[KM];
        float wl[KM];
        block_list<KM>(a, seg, t, true, cl, wl);
#pragma unroll
        for (int r = 0; r < KM; ++r) {
          const int c = cl[r];
          if (!ok || c < 0) continue;
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag)) {
            ok = false;
            break;
          }
          const uint32_t st = sbase + stage * C_STAGE;
          mbar_arrive_expect_tx(full_bar(stage), C_STAGE);
          tma_load_3d(st, &tmX, full_bar(stage), slab * CF, c * CS, b);
          tma_load_3d(st + C_XBOX, &tmX, full_bar(stage), slab * CF + 64, c * CS, b);
          tma_load_3d(st + 2 * C_XBOX, &tmP, full_bar(stage), r * CS, 0, 0);
          ++issued;
          if (++stage == C_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        record_status(a.status, AVEY_ERR_DEVICE_TIMEOUT);
      }
      for (int s = 0; s < C_STAGES; ++s) {
        if (issued > s) {
          const long long last = ((issued - 1 - s) / C_STAGES) * C_STAGES + s;
          cwait_drain(full_bar(s), static_cast<uint32_t>((last / C_STAGES) & 1));
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(CF, CS) | (1u << 15);  // A is MN-major
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
        const long long seg = tile / a.nslab;
        const int t = a.t0 + static_cast<int>(seg % a.nr);
        int cl[KM];
        float wl[KM];
        block_list<KM>(a, seg, t, false, cl, wl);
#pragma unroll
        for (int r = 0; r < KM; ++r) {
          if (!ok || cl[r] < 0) continue;
          if (!mbar_wait(tempty_bar(acc), acc_phase ^ 1u, abort_flag) ||
              !mbar_wait(full_bar(stage), phase, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = sbase + stage * C_STAGE;
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * 64);
#pragma unroll
          for (int kk = 0; kk < CS / 16; ++kk)
            tc_mma_bf16(d_tmem, cdesc_mn(st + 2048u * kk), cdesc_k(st + 2 * C_XBOX + 32u * kk),
                        idesc, kk != 0);
          if (r == 0) {  // + X_t^T: the residual
#pragma unroll
            for (int kk = 0; kk < CS / 16; ++kk)
              tc_mma_bf16(d_tmem, cdesc_mn(st + 2048u * kk), cdesc_k(ibase + 32u * kk), idesc, 1u);
          }
          tc_commit(empty_bar(stage));
          tc_commit(tfull_bar(acc));
          if (++stage == C_STAGES) {
            stage = 0;
            phase ^= 1u;
          }
          if (++acc == C_NACC) {
            acc = 0;
            acc_phase ^= 1u;
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
    const int quarter = warp & 3;      // TMEM lanes = features 32*quarter .. +31 of the slab
    const int half = (warp - 2) >> 2;  // TMEM columns = tokens 32*half .. +31 of the split
    int acc = 0;
    uint32_t acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < a.num_tiles && ok; tile += gridDim.x) {
      const long long seg = tile / a.nslab;
      const int slab = static_cast<int>(tile - seg * a.nslab);
      const int b = static_cast<int>(seg / a.nr);
      const int t = a.t0 + static_cast<int>(seg - static_cast<long long>(b) * a.nr);
      float o[C_TOK];
#pragma unroll
      for (int i = 0; i < C_TOK; ++i) o[i] = 0.f;
      int cl[KM];
      float wl[KM];
      block_list<KM>(a, seg, t, false, cl, wl);
#pragma unroll
      for (int r = 0; r < KM; ++r) {
        if (!ok || cl[r] < 0) continue;
        const float wr = wl[r];
        if (!mbar_wait(tfull_bar(acc), acc_phase, abort_flag)) {
          ok = false;
          continue;
        }
        tc_fence_after();
        float v[C_TOK];
        tmem_ld32(tmem_base + static_cast<uint32_t>(acc * 64 + half * C_TOK) +
                      (static_cast<uint32_t>(quarter * 32) << 16),
                  v);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
#pragma unroll
        for (int i = 0; i < C_TOK; ++i) o[i] = fmaf(wr, v[i], o[i]);
        if (++acc == C_NACC) {
          acc = 0;
          acc_phase ^= 1u;
        }
      }
      if (!ok) break;
      // fp32 out and the split pair: each warp stages its 32 features x 32
      // tokens and writes them with its own three TMA stores (the tensor's
      // bounds clip the feature tail)
      uint8_t *wst = ostage + (warp - 2) * C_WSTG;
      const uint32_t wsa = obase + (warp - 2) * C_WSTG;
      if (lane == 0) bulk_wait_read<0>();  // this warp's previous stores have read it
      __syncwarp();
      {
        float *o32 = reinterpret_cast<float *>(wst);
        bf16 *oh = reinterpret_cast<bf16 *>(wst + C_W32);
        bf16 *ol = reinterpret_cast<bf16 *>(wst + C_W32 + C_W16);
        const bool f32out = a.out != nullptr;
#pragma unroll
        for (int i = 0; i < C_TOK; ++i) {
          const float y = o[i];
          const bf16 h = __float2bfloat16_rn(y);
          if (f32out) o32[i * 32 + lane] = y;
          oh[i * 32 + lane] = h;
          ol[i * 32 + lane] = __float2bfloat16_rn(y - __bfloat162float(h));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        const int orow = static_cast<int>(seg * CS) + half * C_TOK, ox = slab * CF + quarter * 32;
        if (a.out) tma_store_3d(&tmO, wsa, ox, orow, 0);
        if (a.out_hi) {
          tma_store_3d(&tmOh, wsa + C_W32, ox, orow, 0);
          tma_store_3d(&tmOl, wsa + C_W32 + C_W16, ox, orow, 0);
        }
        bulk_commit();
      }
    }
    if (lane == 0) bulk_wait_all();  // this warp's outputs written before exit
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

template <int KM>
avey_status run_compress_tc(const CUtensorMap &mx, const CUtensorMap &mp, const CUtensorMap &mo,
                            const CUtensorMap &moh, const CUtensorMap &mol, const CompArgs &a,
                            int grid, cudaStream_t s) {
  auto kern = compress_tc_kernel<KM>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C_SMEM));
  if (e != cudaSuccess) {
    set_detail("compress_tc: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return AVEY_ERR_CUDA;
  }
  kern<<<grid, C_THR, C_SMEM, s>>>(mx, mp, mo, moh, mol, a);
  AVEY_CHECK_LAUNCH("compress_tc", s);
  return AVEY_OK;
}

}  // namespace

bool compress_tc_supported(int S, int d) { return S == CS && d % 8 == 0; }

avey_status launch_compress_tc(const bf16 *x, int B, int N, int d, int k, int t0, int nr,
                               const int32_t *idx, const float *w, const bf16 *P, float *out,
                               bf16 *hi, bf16 *lo, cudaStream_t s) {
  const int n = (N + CS - 1) / CS;
  CUtensorMap mx, mp;
  const uint64_t rs = static_cast<uint64_t>(d) * 2;
  if (!encode_map(&mx, false, x, d, N, B, rs, rs * N, 64, CS, 128)) return AVEY_ERR_CUDA;
  const uint64_t ps = static_cast<uint64_t>(k + 1) * CS * 2;
  if (!encode_map(&mp, false, P, static_cast<uint64_t>(k + 1) * CS, CS, 1, ps, ps * CS, 64, CS, 128))
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
  // outputs [B*nr*64 rows, d]: fp32 and the bf16 planes, dense boxes of 32 x 32
  CUtensorMap mo, moh, mol;
  const uint64_t orows = static_cast<uint64_t>(B) * nr * CS;
  const uint64_t o4 = static_cast<uint64_t>(d) * 4, o2 = static_cast<uint64_t>(d) * 2;
  if (out && !encode_map(&mo, true, out, d, orows, 1, o4, o4 * orows, 32, C_TOK, 0)) return AVEY_ERR_CUDA;
  if (hi) {
    if (!encode_map(&moh, false, hi, d, orows, 1, o2, o2 * orows, 32, C_TOK, 0)) return AVEY_ERR_CUDA;
    if (!encode_map(&mol, false, lo, d, orows, 1, o2, o2 * orows, 32, C_TOK, 0)) return AVEY_ERR_CUDA;
  }
  // the kernel never uses the map of an output it does not write
  if (!out) mo = moh;
  if (!hi) moh = mol = mo;
  if (k + 1 <= 8) return run_compress_tc<8>(mx, mp, mo, moh, mol, a, grid, s);
  if (k + 1 <= 16) return run_compress_tc<16>(mx, mp, mo, moh, mol, a, grid, s);
  return run_compress_tc<32>(mx, mp, mo, moh, mol, a, grid, s);
}

}  // namespace avey
