/*
 * avey.h -- C ABI of the B200 (sm_100a) Avey-B ranker and neural-processor
 * library (libavey.so).
 *
 * Pages defining the operations (cited by title and section):
 *   [AB-notes] "Avey-B: 把无注意力架构改造成双向编码器" (papernotes.org ICLR 2026
 *              note): 方法详解 整体框架 (splits, MaxSim ranker, top-k,
 *              divide-by-max weights, enricher Z = sigma(XU+b), fuser
 *              f = [Z_h || c(Z_t)] O plus residual); 关键设计 2 (static layer
 *              c = V Z_t, dynamic layer N(Z_t) N(Z_t)^T); 关键设计 3 (eq. 6,
 *              divide by row sum + eps); 关键设计 4 (eq. 8, X_hat = P X_cat,
 *              residual to the split's own tokens).
 *   [AB-sum]   "Avey-B" (paperlayer.ai summary of arXiv 2602.15814v1): §3
 *              Background (ranker, enricher/contextualizer/fuser), §4
 *              (bidirectional, decoupled layers, compression), App. A (ReLU^2
 *              enricher), App. B (S -> D interleaving), App. H (ranker once,
 *              on the initial embeddings).
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers unless a parameter says otherwise.  The
 *     caller allocates and owns every buffer, including workspaces; the
 *     library never allocates device memory and keeps no per-call state.
 *     One exception: avey_rank_static (below) keeps its scratch in a 16 MiB
 *     device array inside the library, held on every GPU that loads it, whose
 *     contents persist from one call to the next.
 *   - Row-major, densely packed tensors unless an leading dimension ("ld",
 *     in elements) is given.  Base addresses must be 16-byte aligned.
 *   - Every call is asynchronous on `stream` (0 = legacy default stream).
 *     Argument errors are detected on the host BEFORE any launch and return
 *     AVEY_ERR_INVALID_ARG / AVEY_ERR_UNSUPPORTED with nothing enqueued.
 *     Launch failures return AVEY_ERR_CUDA.
 *   - Kernel-side failures (a bounded wait that ran out, a failed bounds
 *     check) never trap: the kernel records a code in a device status word
 *     and returns.  Read it with avey_device_status().
 *   - Padding: a sequence of N tokens is cut into n = ceil(N/S) splits of S
 *     tokens; the last split is zero-padded ([AB-notes] 整体框架).  Outputs
 *     that are per token have n*S rows per sequence; the caller keeps the
 *     first N.
 *
 * Types
 *   AVEY_F32    fp32 everywhere (SIMT kernels, fp32 accumulate).
 *   AVEY_BF16   bf16 embeddings and weights; tensor-core contractions with
 *               fp32 accumulation; fp32 residual stream.
 *   AVEY_BF16X2 a "split" activation: an fp32 value x held as two bf16 planes,
 *               hi = bf16(x) and lo = bf16(x - hi), the lo plane directly
 *               after the hi plane (plane stride = rows * ld elements).  Layer
 *               activations use it so that products against bf16 weights
 *               keep about 16 significant bits.
 */
#ifndef AVEY_H_
#define AVEY_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define AVEY_API __attribute__((visibility("default")))
#else
#define AVEY_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *avey_stream_t; /* == cudaStream_t */

typedef enum {
  AVEY_OK = 0,
  AVEY_ERR_INVALID_ARG = 1,    /* null pointer, bad size, misaligned pointer, too-small workspace */
  AVEY_ERR_UNSUPPORTED = 2,    /* valid but not implemented shape/dtype combination */
  AVEY_ERR_CUDA = 3,           /* a CUDA runtime call or launch failed */
  AVEY_ERR_DEVICE_TIMEOUT = 4, /* a kernel's bounded wait ran out (reported by avey_device_status) */
  AVEY_ERR_DEVICE_BOUNDS = 5   /* a kernel's bounds check failed (reported by avey_device_status) */
} avey_status;

typedef enum { AVEY_F32 = 0, AVEY_BF16 = 1, AVEY_BF16X2 = 2 } avey_dtype;

/* Contextualizer kinds: the two Avey-B layers, plus the coupled causal layer
 * of the original (autoregressive) Avey for comparison. */
typedef enum { AVEY_STATIC = 0, AVEY_DYNAMIC = 1, AVEY_COUPLED_CAUSAL = 2 } avey_ctx_kind;

/* avey_rank_ex flags */
enum { AVEY_RANK_UNIDIRECTIONAL = 1 };

/* ------------------------------------------------------------------ ranker --
 * avey_rank: the ranker, run once per forward on the input embeddings
 * ([AB-sum] App. H).
 *   1. N(x) = x / max(||x||_2, 1e-12) per token (pad rows are zero).
 *   2. MaxSim score(t, c) = sum_{i in split t} max_{j in split c} N(x_i).N(x_j)
 *      for every ordered pair of splits of the same sequence (bidirectional:
 *      [AB-sum] §4; definition: [AB-sum] §3, [AB-notes] 整体框架).  The
 *      (n*S) x (n*S) similarity matrix is never materialised.
 *   3. Top-k per target split over c != t, ordered by (score desc, index asc);
 *      w_r = s_r / s_1 so the best selected split has weight exactly 1
 *      ([AB-notes] 整体框架: "divide by the largest").
 *
 * x       [B, N, d], dtype dt (AVEY_F32 or AVEY_BF16), read only.
 * idx     [B, n, k] int32 out: selected splits in rank order; -1 where n-1 < k.
 * w       [B, n, k] fp32 out: normalised weights (0 where idx is -1).
 * scores  [B, n, n] fp32 out, or NULL: the full split-score matrix (diagonal
 *         included), written when non-NULL.
 * ws      device workspace of at least avey_rank_workspace_bytes(...) bytes,
 *         256-byte aligned.  Contents are scratch (undefined afterwards).
 * Constraints: B, N, d, S, k >= 1; d % 8 == 0; k <= 32.  AVEY_BF16 needs S in
 * {16, 32, 64, 128}; AVEY_F32 needs S a power of two <= 128.
 */
AVEY_API avey_status avey_rank(const void *x, avey_dtype dt, int B, int N, int d, int S, int k,
                      int32_t *idx, float *w, float *scores, void *ws, size_t ws_bytes,
                      avey_stream_t stream);

AVEY_API size_t avey_rank_workspace_bytes(avey_dtype dt, int B, int N, int d, int S);

/* avey_rank_ex: avey_rank with flags.  AVEY_RANK_UNIDIRECTIONAL restricts the
 * candidates of target split t to the preceding splits c < t (the ranker of
 * the original Avey; [AB-sum] App. B "Ranker direction" compares both), so
 * split t gets min(k, t) real candidates and the rest are -1 / 0.  Scores are
 * computed for every pair either way.  flags = 0 is avey_rank. */
AVEY_API avey_status avey_rank_ex(const void *x, avey_dtype dt, int B, int N, int d, int S, int k,
                                  uint32_t flags, int32_t *idx, float *w, float *scores, void *ws,
                                  size_t ws_bytes, avey_stream_t stream);

/* avey_rank_static: avey_rank for callers that cannot allocate device memory
 * (a plugin interface that hands over only input and output buffers, or a
 * host that forbids cudaMalloc on the calling path).  The pages have no
 * counterpart: this is a deployment variant of the ranker, not a step of the
 * method.  It computes exactly what avey_rank computes, with the same kernels,
 * but its scratch lives in a fixed device array inside the library
 * (avey_rank_static_max_scratch_bytes(), 16 MiB, held by every GPU that loads
 * the library until the process exits) instead of a caller workspace.
 *   - It allocates nothing.  A shape whose scratch
 *     (avey_rank_workspace_bytes) exceeds the array is rejected with
 *     AVEY_ERR_UNSUPPORTED before anything is enqueued.
 *   - Every call looks up the array's device address on the current device
 *     (cudaGetSymbolAddress, which allocates nothing).  The first call on a
 *     device may load the library's device code there: make that first call
 *     before any stream capture.
 *   - All calls share the array, which keeps the previous call's contents; every
 *     call rewrites what it reads.  Calls whose kernels overlap on the GPU
 *     (e.g. on two unordered streams) race on it: order them.
 * Arguments and constraints as for avey_rank, without scores and workspace. */
AVEY_API avey_status avey_rank_static(const void *x, avey_dtype dt, int B, int N, int d, int S,
                                      int k, int32_t *idx, float *w, avey_stream_t stream);

AVEY_API size_t avey_rank_static_max_scratch_bytes(void);

/* avey_topk: the selection and weights of avey_rank from precomputed split
 * scores ([AB-sum] §3: top-k candidates, weights divided by the largest):
 * per target t, the k candidates c != t (c < t with AVEY_RANK_UNIDIRECTIONAL)
 * of highest score, ties to the lower index, w_r = s_r / max(s_1, 1e-30).
 * scores [B, n, n] fp32 (row t = target t); idx, w [B, n, k] out (idx -1 and
 * w 0 past the available candidates).  Constraints: k <= 32; B*n < 2^31.
 */
AVEY_API avey_status avey_topk(const float *scores, int B, int n, int k, uint32_t flags,
                               int32_t *idx, float *w, avey_stream_t stream);

/* avey_topk_rows: avey_topk for the targets t0 .. t1-1 of every sequence
 * (scores [B, n, n] as above; idx, w [B, t1-t0, k]).  With one long sequence
 * sharded across GPUs, each rank selects for its own targets. */
AVEY_API avey_status avey_topk_rows(const float *scores, int B, int n, int t0, int t1, int k,
                                    uint32_t flags, int32_t *idx, float *w, avey_stream_t stream);

/* avey_maxsim_part: the split scores of avey_rank from one part of the work,
 * for one long sequence sharded across GPUs.  The triangular tile order of
 * the MaxSim kernel (each 256x256 tile on or right of the diagonal gives the
 * scores of its split pairs in both directions) is dealt round-robin into
 * nparts parts; part `part` writes the entries of its tiles and leaves the
 * others untouched.  Every entry belongs to exactly one part, so zeroed score
 * buffers summed over all parts (an all-reduce) give avey_rank's scores bit
 * for bit.  x, ws as for avey_rank (ws >= avey_rank_workspace_bytes);
 * scores [B, n, n] fp32, zeroed by the caller.
 * Constraints: AVEY_BF16, S in {32, 64, 128}; 0 <= part < nparts.
 */
AVEY_API avey_status avey_maxsim_part(const void *x, avey_dtype dt, int B, int N, int d, int S,
                                      int part, int nparts, float *scores, void *ws,
                                      size_t ws_bytes, avey_stream_t stream);

/* ---------------------------------------------------------- compression --
 * avey_compress: neural compression of each split with its retrieved splits
 * plus the residual to the split's own tokens ([AB-notes] 关键设计 4, eq. 8):
 *   X_cat(t) = [X_t ; w_1 X_c1 ; ... ; w_k X_ck]   ((k+1)S x d, rank order)
 *   out(t)   = P X_cat(t) + X_t,   P in R^{S x (k+1)S}, shared by all splits.
 * A candidate index of -1 contributes a zero block.
 *
 * x        [B, N, d] embeddings, dtype dt (AVEY_F32 or AVEY_BF16).
 * idx, w   [B, n, k] from avey_rank (any int32 in [-1, n) is accepted; out of
 *          range indices are rejected on the device as AVEY_ERR_DEVICE_BOUNDS
 *          and their block is treated as zero).
 * P        [S, (k+1)S], dtype dt.
 * out      [B, n*S, d] fp32 out (the residual stream entering layer 0).  For
 *          AVEY_BF16 it may be NULL when out_lowp is given: only the pair is
 *          written (avey_layer_forward can then take x_in = NULL).
 * out_lowp for AVEY_BF16: NULL or an AVEY_BF16X2 pair [2][B*n*S][d] of `out`
 *          (what avey_layer_forward reads as x_in_lowp).  Ignored for F32.
 * Constraints: d % 8 == 0; k <= 32; AVEY_BF16 needs S in {16, 32, 64, 128};
 * AVEY_F32 needs S a power of two <= 64.
 */
AVEY_API avey_status avey_compress(const void *x, avey_dtype dt, int B, int N, int d, int S, int k,
                          const int32_t *idx, const float *w, const void *P, float *out,
                          void *out_lowp, avey_stream_t stream);

/* avey_compress_rows: avey_compress for the target splits t0 .. t1-1 of every
 * sequence: idx, w are [B, t1-t0, k] (as from avey_topk_rows; candidate
 * indices still refer to the whole sequence), out [B, (t1-t0)*S, d] fp32,
 * out_lowp the pair [2][B*(t1-t0)*S][d] or NULL. */
AVEY_API avey_status avey_compress_rows(const void *x, avey_dtype dt, int B, int N, int d, int S,
                                        int k, int t0, int t1, const int32_t *idx, const float *w,
                                        const void *P, float *out, void *out_lowp,
                                        avey_stream_t stream);

/* --------------------------------------------------- uncompressed context --
 * avey_context: the context of every split without neural compression, for
 * the processor variant that contextualizes all (k+1)S tokens of each split
 * ([AB-sum] §4.3, the ablation behind the 4.37x throughput figure; the
 * tensor is the compressor's input of eq. 8, [AB-notes] 关键设计 4):
 *   ctx(b, t) = [X_t ; w_1 X_c1 ; ... ; w_k X_ck]   ((k+1)S x d, rank order)
 * The target block is unweighted; a candidate of -1 and the pad rows of a
 * ragged last split are zero rows.
 *
 * x, idx, w as for avey_compress (out of range indices are rejected on the
 *          device as AVEY_ERR_DEVICE_BOUNDS and their block is zero).
 * out      [B, n, (k+1)S, d] fp32 (caller-owned).
 * out_lowp for AVEY_BF16: NULL or an AVEY_BF16X2 pair [2][B*n*(k+1)S][d] of
 *          `out`.  Ignored for F32.
 * The processor then runs avey_layer_forward on T = B*n*(k+1)S tokens with
 * S = (k+1)S (one block per split); rows [0, S) of each block are the split's
 * output.  Constraints: d % 8 == 0; k <= 32.
 */
AVEY_API avey_status avey_context(const void *x, avey_dtype dt, int B, int N, int d, int S, int k,
                                  const int32_t *idx, const float *w, float *out, void *out_lowp,
                                  avey_stream_t stream);

/* ------------------------------------------------------------ static mix --
 * avey_static_mix: the static contextualizer of one layer on `blocks`
 * independent split blocks of S tokens ([AB-notes] 关键设计 2):
 *   c = V Z_t     (V: S x S, shared by all blocks; identity activation, no bias)
 * V    [S, S] row-major, fp32 for AVEY_F32, bf16 for AVEY_BF16X2.
 * zt, out: layouts as for avey_dynamic_mix (out may alias zt exactly).
 * Constraints: S in {16, 32, 64, 128} for AVEY_BF16X2 (a power of two <= 64
 * for F32); mt % 8 == 0 and ld % 8 == 0 for AVEY_BF16X2.
 */
AVEY_API avey_status avey_static_mix(const void *V, const void *zt, int64_t ld_zt, avey_dtype dt,
                                     int blocks, int S, int mt, void *out, int64_t ld_out,
                                     avey_stream_t stream);

/* ----------------------------------------------------------- dynamic mix --
 * avey_dynamic_mix: the dynamic contextualizer of one layer on `blocks`
 * independent split blocks of S tokens ([AB-notes] 关键设计 2 and 3):
 *   G_ij  = N(z_i) . N(z_j)              (cosine, N(z) = z / max(||z||, 1e-12))
 *   Gt_ij = G_ij / (sum_j G_ij + eps)    (eq. 6)
 *   c     = Gt Z_t                        (identity activation, no bias)
 * zt   block b, token i, feature f at zt[(b*S + i) * ld_zt + f], f < mt.
 *      AVEY_F32: fp32.  AVEY_BF16X2: split pair, lo plane at
 *      zt + blocks*S*ld_zt elements.
 * out  same layout and dtype with ld_out (lo plane at out + blocks*S*ld_out).
 *      out may alias zt exactly (in place); partial overlap is not allowed.
 * Constraints: S in {16, 32, 64, 128} for AVEY_BF16X2 (a power of two <= 64
 * for F32);
 * mt % 8 == 0 and ld % 8 == 0 for AVEY_BF16X2; eps >= 0.
 */
AVEY_API avey_status avey_dynamic_mix(const void *zt, int64_t ld_zt, avey_dtype dt, int blocks, int S,
                             int mt, float eps, void *out, int64_t ld_out, avey_stream_t stream);

/* ----------------------------------------------------------------- layer --
 * avey_layer_forward: one neural-processor layer on T = blocks * S tokens
 * ([AB-notes] 整体框架, 关键设计 2-3; [AB-sum] §3, App. A):
 *   xin = prenorm ? x / sqrt(mean(x^2) + 1e-6) : x   (per token; see below)
 *   Z   = relu(xin U + b)^2                          (enricher, ReLU^2)
 *   Z_h = Z[:, :m_h],  Z_t = Z[:, m_h:]              (head bypass / tail)
 *   c   = V Z_t (static) or Gt Z_t (dynamic), per split of S tokens; for
 *         AVEY_COUPLED_CAUSAL, c = M Z_t with M_ij = V_ij N(z_i).N(z_j) for
 *         j <= i and 0 otherwise (the original Avey's coupled contextualizer,
 *         [AB-notes] 关键设计 2, with its causal mask; no row normalisation)
 *   x'  = x + [Z_h || c] O                           (fuser + residual)
 * `prenorm` is an option of this library, not of the pages: a gain-free RMS
 * norm of the enricher input that keeps deep stacks finite.  It leaves the
 * residual path untouched.
 *
 * Weights (dtype = dt: AVEY_F32, or AVEY_BF16 for the tensor-core path):
 *   Ut [m, d]  the enricher matrix U stored transposed (row f holds U[:, f])
 *   bU [m]     fp32 enricher bias (fp32 for both dtypes)
 *   V  [S, S]  static map (AVEY_STATIC, AVEY_COUPLED_CAUSAL), NULL for AVEY_DYNAMIC
 *   Ot [d, m]  the fuser matrix O stored transposed (row q holds O[:, q])
 * Activations:
 *   x_in      [T, d] fp32 residual stream in.  For AVEY_BF16 it may be NULL
 *             when x_in_lowp is given: the residual is then hi + lo of the
 *             pair (about 16 significant bits; exact as fp32 arithmetic).
 *   x_in_lowp AVEY_BF16 only: NULL or the AVEY_BF16X2 pair of x_in (as
 *             written by avey_compress / the previous layer).  When NULL the
 *             pair is built in the workspace.
 *   x_out     [T, d] fp32 out (may alias x_in exactly).  For AVEY_BF16 it may
 *             be NULL when x_out_lowp is given: only the pair is written.
 *   x_out_lowp AVEY_BF16 only: NULL or an AVEY_BF16X2 pair [2][T][d] out (may
 *             alias x_in_lowp exactly).
 *   A stack that passes the pair alone between layers writes fp32 only after
 *   its last layer: per token and layer it moves 4 d bytes fewer.
 *   ws        >= avey_layer_workspace_bytes(...) bytes, 256-byte aligned.
 * Constraints: T % S == 0; d, m, m_h multiples of 8 with 0 < m_h < m;
 * S in {16, 32, 64, 128} for AVEY_BF16, and also 256 or 512 for static and
 * dynamic layers (the blocks of (k+1)S tokens of the uncompressed processor,
 * see avey_context; these need m_h % 64 == 0, and m - m_h <= 1024 for a
 * dynamic layer); a power of two <= 64 for F32; eps >= 0.
 */
typedef struct {
  avey_ctx_kind kind;
  int d, m, m_h, S;
  float eps;
  int prenorm;
  const void *Ut;
  const float *bU;
  const void *V;
  const void *Ot;
} avey_layer_params;

AVEY_API avey_status avey_layer_forward(const avey_layer_params *p, avey_dtype dt, int T,
                               const float *x_in, const void *x_in_lowp, float *x_out,
                               void *x_out_lowp, void *ws, size_t ws_bytes,
                               avey_stream_t stream);

/* avey_layer_forward_ex: avey_layer_forward with the per-row prenorm scales
 * r = 1 / sqrt(mean(x^2) + 1e-6) passed between the layers of a stack, so that
 * no layer re-reads its input to compute them.  The pages define the layer;
 * handing its scales over is a property of this implementation only.
 * x_in_rms   [T] fp32 or NULL: the scales of x_in (as a previous layer's
 *            x_out_rms wrote them).  Used in place of computing them when
 *            p->prenorm; ignored otherwise.
 * x_out_rms  [T] fp32 or NULL: also write the scales of x_out, from its fp32
 *            values before the split (on the bf16 path the fuser computes
 *            them in its epilogue; on the fp32 path a separate kernel does).
 *            Must not be x_in_rms.
 * Both 4-byte aligned.  Everything else as avey_layer_forward, which is this
 * call with both NULL.  The scales from x_out_rms equal a recomputation from
 * x_out's split pair to within float rounding of the sum (about 1e-6
 * relative), not bit for bit. */
AVEY_API avey_status avey_layer_forward_ex(const avey_layer_params *p, avey_dtype dt, int T,
                                           const float *x_in, const void *x_in_lowp,
                                           const float *x_in_rms, float *x_out, void *x_out_lowp,
                                           float *x_out_rms, void *ws, size_t ws_bytes,
                                           avey_stream_t stream);

/* Workspace of avey_layer_forward for S <= 128 (any kind). */
AVEY_API size_t avey_layer_workspace_bytes(avey_dtype dt, int T, int d, int m, int prenorm);

/* Workspace of avey_layer_forward for any supported S and kind: a dynamic
 * layer over blocks of 256 or 512 tokens also holds each block's Gt (as a
 * bf16 split pair, 4 S^2 bytes per block) and two fp32 scales per token. */
AVEY_API size_t avey_layer_workspace_bytes_ex(avey_dtype dt, int T, int d, int m, int prenorm, int S,
                                              avey_ctx_kind kind);

/* ------------------------------------------------------------- utilities --
 * avey_device_status: synchronises `stream`, returns the first kernel-side
 * failure recorded since the previous call (AVEY_ERR_DEVICE_TIMEOUT or
 * AVEY_ERR_DEVICE_BOUNDS) or AVEY_OK, and clears it.  Returns AVEY_ERR_CUDA
 * if the synchronisation itself fails.
 */
AVEY_API avey_status avey_device_status(avey_stream_t stream);

/* avey_status_string: static, never NULL. */
AVEY_API const char *avey_status_string(avey_status s);

/* avey_last_error_detail: a static description of the last host-side
 * rejection or CUDA error in this thread (empty string if none). */
AVEY_API const char *avey_last_error_detail(void);

/* avey_selftest_wait_timeout: diagnostic with no counterpart on the pages.
 * Launches one warp that waits, through the same bounded wait the tcgen05
 * kernels use, on a barrier nothing arrives on, for limit_us microseconds
 * (1 .. 2e6); the wait then gives up, records AVEY_ERR_DEVICE_TIMEOUT in the
 * device status word and the kernel returns.  The next avey_device_status()
 * reports it; the context stays usable. */
AVEY_API avey_status avey_selftest_wait_timeout(uint32_t limit_us, avey_stream_t stream);

/* Kernel trace: a measurement hook with no counterpart on the pages.
 * avey_trace_begin records a start event on `stream`; then, until
 * avey_trace_end, every kernel the library launches records the next event
 * on its own launch stream right after it is enqueued, and the library keeps
 * the kernel's name.  The events belong to the library: they are created on
 * the current device by the first trace that needs them (no device memory),
 * reused by later traces, and held until the process exits; all traces must
 * run on that device (AVEY_ERR_UNSUPPORTED otherwise).
 *   capacity  1 <= capacity <= 4096 launches are timed; later launches are
 *             counted but record nothing.
 * avey_trace_begin returns AVEY_ERR_INVALID_ARG for a bad capacity or while a
 * trace is already active (one trace per process, shared by all host
 * threads), AVEY_ERR_CUDA when an event cannot be created or recorded.
 * avey_trace_end returns the number of launches seen (which may exceed the
 * capacity), or -1 if no trace was active or an event record failed (detail
 * in avey_last_error_detail).
 * After avey_trace_end, for traced launch i < min(count, capacity):
 *   avey_trace_kernel_name(i)  its kernel (a string owned by the library,
 *                              valid until the next trace begins), else NULL;
 *   avey_trace_kernel_ms(i, &ms)  the device time between the event before it
 *                              (the start, or launch i-1's) and its own; on one
 *                              stream that is the kernel's duration.  The
 *                              events must have completed (synchronise the
 *                              stream first), else AVEY_ERR_CUDA. */
AVEY_API avey_status avey_trace_begin(int capacity, avey_stream_t stream);
AVEY_API int avey_trace_end(void);
AVEY_API const char *avey_trace_kernel_name(int i);
AVEY_API avey_status avey_trace_kernel_ms(int i, float *ms);

/* avey_kernel_launches: number of kernels this library has launched since it
 * was loaded, in this process (all threads). */
AVEY_API uint64_t avey_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* AVEY_H_ */
