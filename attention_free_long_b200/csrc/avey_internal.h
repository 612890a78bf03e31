// avey_internal.h -- launchers shared between the translation units of
// libavey.so.  Not part of the public ABI (include/avey.h is).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "avey.h"

namespace avey {

using bf16 = __nv_bfloat16;

// ---- tcgen05 contractions (avey_tc.cu) ----

// MaxSim split scores from the raw embeddings x [B, N, d] bf16 and the
// inverse row norms inv_norm [B, rs_ld] (rs_ld >= R rounded up to 256, zero
// past N); R = n*S.  Full tile grid on one CTA per SM, for S = 16.
avey_status launch_maxsim_tc(const bf16 *x, const float *inv_norm, int B, int N, int R, int rs_ld,
                             int d, int S, int n, float *scores, cudaStream_t s);

// The same scores from 256 x 256 tiles on CTA pairs (tcgen05 cta_group::2),
// avey_maxsim2.cu; S in {32, 64, 128}, rs_ld >= R rounded up to 256.
// part / nparts: compute only the tiles t with t % nparts == part (the others'
// score entries are left untouched); every entry comes from exactly one tile.
avey_status launch_maxsim_pair(const bf16 *x, const float *inv_norm, int B, int N, int R, int rs_ld,
                               int d, int S, int n, float *scores, cudaStream_t s, int part = 0,
                               int nparts = 1);

// Enricher: Z = relu(scale_row * (X U) + b)^2, X given as a split pair
// (xhi, xlo) [T, d]; Ut [m, d]; writes the split pair of Z (zhi, zlo) [T, m].
// inv_rms may be null (scale 1).
avey_status launch_enrich_tc(const bf16 *xhi, const bf16 *xlo, int T, int d, const bf16 *Ut,
                             int m, const float *bias, const float *inv_rms, bf16 *zhi,
                             bf16 *zlo, cudaStream_t s);

// Fuser: x_out = x_in + A O, A given as a split pair (ahi, alo) [T, m];
// Ot [d, m]; writes fp32 x_out and (optionally) its split pair.
// With chi / clo given, activation columns [k_split, m) are read from the
// split pair c [T, m - k_split] instead of (ahi, alo); k_split % 64 == 0.
// Residual: x_in (fp32) or, when x_in is null, the pair (xin_hi, xin_lo).
// Output: x_out (fp32) and/or the pair (xo_hi, xo_lo); either may be null.
// rms_out (nullable): also 1 / sqrt(mean(x_out^2) + 1e-6) per row, from the
// fp32 output values (the next layer's prenorm scale).
avey_status launch_fuse_tc(const bf16 *ahi, const bf16 *alo, int T, int m, const bf16 *Ot, int d,
                           const float *x_in, const bf16 *xin_hi, const bf16 *xin_lo, float *x_out,
                           bf16 *xo_hi, bf16 *xo_lo, cudaStream_t s, const bf16 *chi = nullptr,
                           const bf16 *clo = nullptr, int k_split = 0, float *rms_out = nullptr);

// Compression on tcgen05 (avey_compress_tc.cu) for S = 64 and 128, targets
// t0 .. t0+nr-1 (idx, w, out as for avey_compress_rows); the split-size
// mma.sync kernel covers S = 16 and 32.
bool compress_tc_supported(int S, int d);
avey_status launch_compress_tc(const bf16 *x, int B, int N, int d, int S, int k, int t0, int nr,
                               const int32_t *idx, const float *w, const bf16 *P, float *out,
                               bf16 *hi, bf16 *lo, cudaStream_t s);

// ---- ranker pieces (avey_rank.cu) ----
// Shape and dtype checks of the ranker entry points (avey_rank.cu); fn names
// the entry point in the error detail.
avey_status check_rank_shape(const char *fn, avey_dtype dt, int B, int N, int d, int S, int k);

avey_status launch_normalize(const void *x, avey_dtype dt, int B, int N, int d, int S, void *xhat,
                             cudaStream_t s);
avey_status launch_inv_norms(const bf16 *x, int B, int N, int d, int rs_ld, float *inv,
                             cudaStream_t s);
avey_status launch_topk(const float *scores, int B, int n, int k, int causal, int32_t *idx,
                        float *w, cudaStream_t s);
// Targets t0 .. t0+nr-1 of every sequence; idx, w are [B, nr, k].
avey_status launch_topk_rows(const float *scores, int B, int n, int t0, int nr, int k, int causal,
                             int32_t *idx, float *w, cudaStream_t s);

// ---- mixes (avey_mix.cu) ----
avey_status launch_static_mix_x2(const bf16 *V, const bf16 *zt, int64_t ld, int blocks, int S,
                                 int mt, int64_t plane, bf16 *out, int64_t ld_out,
                                 int64_t plane_out, cudaStream_t s);
avey_status launch_dynamic_mix_x2(const bf16 *zt, int64_t ld_zt, int64_t plane_zt, bf16 *out,
                                  int64_t ld_out, int64_t plane_out, int blocks, int S, int mt,
                                  float eps, cudaStream_t s);
// Coupled causal contextualizer (original Avey): c = (V * cos, j <= i) Z_t.
avey_status launch_coupled_mix_x2(const bf16 *V, const bf16 *zt, int64_t ld_zt, int64_t plane_zt,
                                  bf16 *out, int64_t ld_out, int64_t plane_out, int blocks, int S,
                                  int mt, cudaStream_t s);
avey_status launch_coupled_mix_f32(const float *V, const float *zt, int64_t ld_zt, float *out,
                                   int64_t ld_out, int blocks, int S, int mt, cudaStream_t s);
avey_status launch_static_mix_f32(const float *V, const float *zt, int64_t ld_zt, float *out,
                                  int64_t ld_out, int blocks, int S, int mt, cudaStream_t s);
avey_status launch_dynamic_mix_f32(const float *zt, int64_t ld_zt, float *out, int64_t ld_out,
                                   int blocks, int S, int mt, float eps, cudaStream_t s);

// ---- mixes over long blocks of 256 or 512 tokens (avey_mix_long.cu) ----
// In place on the split pair Z_t (hi at zt, lo at zt + plane).  The dynamic
// mix needs long_dynamic_ws_bytes(blocks, SL) bytes of workspace.
size_t long_dynamic_ws_bytes(int blocks, int SL);
// Dynamic Gt of every block (bf16 split pair in the workspace, hi at ws, lo
// at ws + blocks*SL*SL elements) without the apply step.
avey_status launch_long_dynamic_gt(const bf16 *zt, int64_t ld, int blocks, int SL, int mt, float eps,
                                   void *ws, cudaStream_t s);
// c = A Z_t over blocks of SL in {256, 512} tokens on tcgen05 (avey_mix_tc.cu):
// A = the bf16 [SL, SL] map shared by all blocks (a_lo null, a_batched false)
// or every block's Gt pair (a_batched true); Z_t a split pair with row stride
// ldz; c written as a split pair [blocks*SL, mt] (row stride mt) to chi / clo.
// The hi-plane Gram of every block, scaled to Gt (inv_n, inv_d per token from
// the dynamic prep) and written as a split pair: gt [blocks][SL][SL], lo plane
// at gt + blocks*SL*SL (avey_mix_tc.cu).
avey_status launch_long_gram_tc(const bf16 *zhi, int64_t ldz, int blocks, int SL, int mt,
                                const float *inv_n, const float *inv_d, bf16 *gt, cudaStream_t s);
avey_status launch_long_mix_tc(const bf16 *a_hi, const bf16 *a_lo, bool a_batched, const bf16 *zhi,
                               const bf16 *zlo, int64_t ldz, int blocks, int SL, int mt, bf16 *chi,
                               bf16 *clo, cudaStream_t s);
}  // namespace avey
