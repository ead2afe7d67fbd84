/*
 * velox.h -- C ABI of the B200 (sm_100a) routed block-sparse attention path.
 *
 * The path is the hot loop of Velox, a training-free router for the
 * history attention of chunked video-diffusion world models ("Velox: Spatial
 * Memory Makes Long-context World Models Efficient", project page
 * velox-world.com, "02 · Method"; digest of arXiv 2610.22311 on
 * paper.rainbus.top, "Core method" and "Method steps"):
 *
 *   1. velox_gilbert_order      global-aligned Gilbert token order, block ids,
 *                               26-neighbour safeguard blocks;
 *   2. velox_block_importance   p_{i,r} = softmax_r(scale * qbar_i . kbar_r);
 *   3. velox_route_build        soft geometry fusion, minimal cumulative-mass
 *                               prefix capped at K_cov / K_unc, reserved
 *                               previous chunk, appended safeguards;
 *   4. velox_block_sparse_attn  online-softmax attention over only the routed
 *                               128-token KV tiles (tcgen05 / TMEM / TMA).
 *
 * Around it: velox_two_phase_attn (routed history plus the current chunk's
 * own tiles under one softmax), velox_slab_overlap and velox_coverage (the
 * geometric inputs g and the coverage flags), velox_route_audit (the
 * geometry-model consistency counts), velox_thw_linear_order (the raster
 * order the pages compare the Gilbert order with), velox_slab_table and
 * velox_multiwarp (the history-side geometry: frustum slabs from depth maps,
 * the recency-priority multiwarp depth of the current frames),
 * velox_route_schedule (longest-route-first row order),
 * velox_block_importance_noalloc, velox_wait_selftest (the bounded waits
 * driven to their limit) and velox_clock_probe (the SM clock seen from
 * inside the GPU, for measurement).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every pointer argument is a DEVICE pointer, owned by the caller, unless
 *   the argument says "host".  The library never allocates, frees or keeps
 *   caller memory; it keeps no state between calls except a per-device
 *   cache of device attributes and one exception: the fixed device array of
 *   VELOX_NOALLOC_SCRATCH_BYTES and its cached address, used only by
 *   velox_block_importance_noalloc.
 * - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *   default stream) and may be issued from several host threads.
 * - Tensors are dense and contiguous in the layouts stated.  bf16 values are
 *   raw IEEE bfloat16 bit patterns (velox_bf16).
 * - Host-detectable errors (null pointers, non-positive or inconsistent
 *   sizes, unsupported head_dim / block size, too-small capacity or
 *   workspace) return a status before anything is launched.  A CUDA launch
 *   error returns VELOX_ERR_CUDA.
 * - Errors that only the device can see (a route id out of range or
 *   repeated, a capacity overflow, a bounded wait that gave up) are OR-ed
 *   into *dev_status, one int32 in device memory that the caller zeroes
 *   beforehand (VELOX_DEV_* bits).  The offending tile or row is skipped;
 *   no kernel traps or reads out of bounds.
 */
#ifndef VELOX_H_
#define VELOX_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define VELOX_API __attribute__((visibility("default")))
#else
#define VELOX_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t velox_bf16;                 /* raw bfloat16 bits          */
typedef struct CUstream_st *velox_stream_t;  /* == cudaStream_t            */

typedef enum {
  VELOX_OK = 0,
  VELOX_ERR_INVALID_ARG = 1,  /* null pointer, bad size, inconsistent args */
  VELOX_ERR_UNSUPPORTED = 2,  /* head_dim/block size/lattice not supported */
  VELOX_ERR_WORKSPACE = 3,    /* workspace missing or too small            */
  VELOX_ERR_CAPACITY = 4,     /* R_max / S_max cannot hold the output      */
  VELOX_ERR_DEVICE = 5,       /* no usable sm_100 device                   */
  VELOX_ERR_TIMEOUT = 6,      /* reserved: a bounded device wait gave up   */
  VELOX_ERR_CUDA = 7          /* a CUDA runtime call or launch failed      */
} velox_status;

/* Bits OR-ed into *dev_status by the kernels. */
#define VELOX_DEV_BAD_ROUTE_ID   0x01  /* route id < 0 or >= M: tile skipped   */
#define VELOX_DEV_DUP_ROUTE_ID   0x02  /* id repeated in one route: skipped    */
#define VELOX_DEV_ROUTE_LEN      0x04  /* route_len < 0 or > R_max: row zeroed */
#define VELOX_DEV_NBR_OVERFLOW   0x08  /* more neighbours than S_max: cut      */
#define VELOX_DEV_BAD_SAFEGUARD  0x10  /* nbr/ref id outside [0, M): ignored   */
#define VELOX_DEV_WAIT_TIMEOUT   0x20  /* bounded mbarrier wait gave up        */
#define VELOX_DEV_ROUTE_CAPACITY 0x40  /* route row longer than R_max: cut     */
#define VELOX_DEV_BAD_ROW_ORDER  0x80  /* row_order entry outside [0, H*N)      */
#define VELOX_DEV_BAD_CAMERA     0x100 /* camera index outside [0, n_cams)       */
#define VELOX_DEV_BAD_CELL       0x200 /* block cell outside the lattice / frames  */

/* Supported sizes of the importance and attention calls. */
#define VELOX_HEAD_DIM   128
#define VELOX_BLOCK_TOK  128
#define VELOX_MAX_BLOCKS 65536   /* max history blocks M per head            */
#define VELOX_MAX_ROUTE  4096    /* max R_max (routed attention), k_cov, k_unc */

/* Route hyper-parameters (onedev.kr summary, "How it differs": tau = 0.1,
 * g_ref = 0.2, lambda = 2, K_cov = 80, K_unc = 150).  theta_* are the
 * cumulative-mass thresholds of covered / uncovered rows (the pages give no
 * value; 0.9 is the default of the bundled workloads). */
typedef struct {
  float lambda;     /* fusion strength; the multiplier is 1 + lambda * g^      */
  float tau;        /* overlap noise floor: g^ = 0 unless g > tau              */
  float g_ref;      /* overlap normaliser: g^ = min(g / g_ref, 1)              */
  float theta_cov;  /* mass threshold, covered rows                            */
  float theta_unc;  /* mass threshold, uncovered rows                          */
  int32_t k_cov;    /* budget cap (reserved blocks included), covered rows     */
  int32_t k_unc;    /* budget cap (reserved blocks included), uncovered rows   */
} velox_route_params;

/* Human-readable text of a status; never NULL. */
VELOX_API const char *velox_status_string(velox_status s);

/* ABI version of this header (major * 100 + minor): 104. */
VELOX_API int velox_abi_version(void);

/*
 * velox_gilbert_order -- global-aligned Gilbert order, block ids and the
 * 26-neighbour safeguard table.
 *
 * Defined by: project page, "02 · Method", "Keeping neighbours adjacent in
 * the block order" and figure "Incremental Gilbert order"; digest,
 * "Prerequisites", "Gilbert space-filling curve", and "Method steps", Eq. 14.
 *
 * The lattice has n_chunks chunks of T latent frames of H x W tokens; global
 * frame f = chunk * T + t; cell index c = (f * H + y) * W + x.  Each frame is
 * walked by the 2-D generalised Hilbert (Gilbert) curve from (0,0) to
 * (W-1,0), mirrored in x on odd global frames, frames in order:
 *   rank(f, y, x) = f*H*W + r2[y][f odd ? W-1-x : x].
 * Block id = rank / b_tok.  Requires W >= H, not (W odd and H even), and
 * T*H*W % b_tok == 0 (blocks never straddle chunks); else UNSUPPORTED.
 *
 * Outputs (each nullable; int32, n_cells = n_chunks*T*H*W):
 *   rank_of_cell[n_cells], cell_of_rank[n_cells], block_of_cell[n_cells].
 * Safeguards of the N = T*H*W/b_tok query blocks of chunk q_chunk: history
 * block u is listed for query block i when u != i, some token of u is within
 * Chebyshev distance 1 of some token of i in (f, y, x), and
 * cache_first_block <= u < cache_first_block + n_cache_blocks; it is written
 * as the cache id u - cache_first_block.  nbr_ids[N][S_max] (ascending, -1
 * padded) and nbr_cnt[N]; both null to skip.  More than S_max neighbours:
 * the S_max lowest are kept and VELOX_DEV_NBR_OVERFLOW is set.
 * dev_status may be null only when nbr_ids is null.
 */
VELOX_API velox_status velox_gilbert_order(int T, int H, int W, int n_chunks, int b_tok,
                                 int q_chunk, int cache_first_block,
                                 int n_cache_blocks, int32_t *rank_of_cell,
                                 int32_t *cell_of_rank, int32_t *block_of_cell,
                                 int32_t *nbr_ids, int32_t *nbr_cnt, int S_max,
                                 int32_t *dev_status, velox_stream_t stream);

/*
 * velox_thw_linear_order -- the THW-linear (raster) order that the pages set
 * against the global Gilbert order, with the same outputs.
 *
 * Defined by: project page, figure "THW-linear against global Gilbert order"
 * (toy latent H = 3, W = 4, block size 2) and "Keeping neighbours adjacent
 * in the block order".
 *
 * rank(f, y, x) = (f * H + y) * W + x: the rank of a cell is its cell index,
 * a block is b_tok consecutive raster cells.  Arguments, layouts, the
 * safeguard definition and errors are those of velox_gilbert_order, except
 * that any H and W are accepted (T*H*W % b_tok == 0 still required).
 */
VELOX_API velox_status velox_thw_linear_order(int T, int H, int W, int n_chunks, int b_tok,
                                              int q_chunk, int cache_first_block,
                                              int n_cache_blocks, int32_t *rank_of_cell,
                                              int32_t *cell_of_rank, int32_t *block_of_cell,
                                              int32_t *nbr_ids, int32_t *nbr_cnt, int S_max,
                                              int32_t *dev_status, velox_stream_t stream);

/*
 * velox_workspace_size -- bytes of device workspace that
 * velox_block_importance and velox_route_build need for these sizes
 * (one buffer serves both; 256-byte aligned).  bytes: host pointer.
 */
VELOX_API velox_status velox_workspace_size(int H, int N, int M, int d, size_t *bytes);

/*
 * velox_block_importance -- per-head block importance.
 *
 * Defined by: digest, "Method steps", step four (Eq. 9); onedev.kr summary,
 * "How it differs"; project page, "02 · Method", glossary entry for p.
 *
 *   qbar[h][i] = mean of the b_tok query tokens of block i   (fp32 accum.)
 *   kbar[h][r] = mean of the b_tok key tokens of block r
 *   p[h][i][r] = exp(l_r - max_r l) / sum_r exp(l_r - max_r l),
 *                l_r = scale * qbar[h][i] . kbar[h][r]
 *
 * Q [H][N*b_tok][d] bf16, K [H][M*b_tok][d] bf16 (Gilbert token order,
 * head-major), p [H][N][M] fp32 out.  d == b_tok == 128.  ws: device
 * workspace of at least velox_workspace_size() bytes.
 */
VELOX_API velox_status velox_block_importance(const velox_bf16 *Q, const velox_bf16 *K,
                                    int H, int N, int M, int d, int b_tok,
                                    float scale, float *p, void *ws,
                                    size_t ws_bytes, velox_stream_t stream);

/* Size of the fixed device scratch of velox_block_importance_noalloc. */
#define VELOX_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)

/*
 * velox_block_importance_noalloc -- velox_block_importance for callers that
 * cannot allocate device memory.
 *
 * The pages have no counterpart to this call: it serves users of the
 * library, not the method.  Some callers cannot call cudaMalloc: a host
 * framework that budgets all device memory up front and gives its plugins
 * no allocator, or a latency-critical loop that cannot take the device-wide
 * synchronisation of cudaMalloc / cudaFree.  This call takes no workspace and
 * allocates nothing; the block means live in one fixed array of
 * VELOX_NOALLOC_SCRATCH_BYTES bytes inside the library, which every GPU that
 * loads the library holds until the process exits.
 *
 * Arguments, layouts, result and device errors as velox_block_importance,
 * without ws / ws_bytes.  Limit: H * (N + M) * d * 4 bytes must fit in the
 * array (H * (N + M) <= 131072 at d = 128); larger sizes return
 * VELOX_ERR_WORKSPACE before any launch.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress, which may load
 * the library's device code) and caches it for the device's current context;
 * make that first call before any stream capture.  cudaDeviceReset (or
 * anything else that replaces the device's primary context) discards the
 * cache: the next call looks the address up again, so it too belongs before
 * any capture.  Every call on a device shares the one array and leaves its
 * contents behind: calls that overlap on the GPU (other streams, unordered
 * host threads) race on it.
 */
VELOX_API velox_status velox_block_importance_noalloc(const velox_bf16 *Q, const velox_bf16 *K,
                                                      int H, int N, int M, int d, int b_tok,
                                                      float scale, float *p,
                                                      velox_stream_t stream);

/*
 * velox_route_build -- soft geometry fusion and route materialisation.
 *
 * Defined by: project page, "02 · Method", fusion formula
 * p~ ~ p (1 + lambda g^), g^ = [g > tau] min(g / g_ref, 1), and "Covered and
 * uncovered blocks"; digest, "Core method" (Eq. 11) and "Method steps"
 * (Eq. 12-14); onedev.kr summary, "How it differs".
 *
 * Per row (h, i):
 *   w_r = covered[i] ? p_r (1 + lambda g^_{i,r}) : p_r        (fp64)
 *   s_r = covered[i] ? w_r / sum_r' w_r' : p_r                 (fp64)
 *   walk: reserved blocks [prev_begin, prev_begin+prev_count) first, then
 *   the others by w descending (ties: lower id); take blocks while
 *   count < K (K_cov / K_unc) and cumulative s < theta (theta_cov /
 *   theta_unc); reserved blocks are always taken.
 *   extras = (nbr_ids[i][0..nbr_cnt[i]) U ref_ids) minus the budget.
 * Output row: the budget ids ascending, then the extras ascending, each id
 * once; route_len[h][i] = total, route_nbudget[h][i] = budget count; the
 * rest of the row is -1.
 *
 * p [H][N][M] fp32, g [N][M] fp32 (shared by all heads), covered [N] uint8,
 * nbr_ids [N][S_max] / nbr_cnt [N] int32 (both null, or S_max = 0, for no
 * neighbours), ref_ids [n_ref] int32 (null when n_ref = 0).
 * route_ids [H][N][R_max] int32, route_len / route_nbudget [H][N] int32.
 * R_max must be >= min(M, max(k_cov, k_unc, prev_count) + S_max + n_ref);
 * 0 <= k_cov, k_unc <= VELOX_MAX_ROUTE; M <= VELOX_MAX_BLOCKS.  p must be
 * finite and non-negative.
 * Safeguard ids outside [0, M) are ignored and flag VELOX_DEV_BAD_SAFEGUARD.
 * ws: device workspace of at least velox_workspace_size() bytes.
 */
VELOX_API velox_status velox_route_build(const float *p, const float *g,
                               const uint8_t *covered,
                               const velox_route_params *prm, /* host */
                               int prev_begin, int prev_count,
                               const int32_t *nbr_ids, const int32_t *nbr_cnt,
                               int S_max, const int32_t *ref_ids, int n_ref,
                               int H, int N, int M, int32_t *route_ids,
                               int32_t *route_len, int32_t *route_nbudget,
                               int R_max, void *ws, size_t ws_bytes,
                               int32_t *dev_status, velox_stream_t stream);

/*
 * velox_route_schedule -- the order in which velox_block_sparse_attn should
 * take its rows: longest route first (ties keep ascending row order).
 *
 * The pages have no counterpart to this call: it is a launch-order hint for
 * the attention kernel (long rows first, so the last wave of CTAs is made of
 * short rows).  It changes no result.
 *
 * route_len [rows] int32 (values outside [0, R_max] count as 0), row_order
 * [rows] int32 out: a permutation of 0 .. rows-1.  0 < R_max <=
 * VELOX_MAX_ROUTE.
 */
VELOX_API velox_status velox_route_schedule(const int32_t *route_len, int rows, int R_max,
                                            int32_t *row_order, velox_stream_t stream);

/*
 * velox_block_sparse_attn -- attention over routed KV tiles.
 *
 * Defined by: digest, "Core method" (Eq. 15) and "Novelty"; project page,
 * "Why the route is a block, not a token"; onedev.kr summary, "How to use".
 *
 * For head h, query block i and each of its b_tok query tokens q:
 *   O[h][i*b+t] = sum_u softmax_u(softmax_scale * q . k_u) v_u
 * over the tokens u of the tiles route_ids[h][i][0 .. route_len[h][i]),
 * tile r covering key/value tokens [r*b_tok, (r+1)*b_tok) of head h.
 * lse[h][i*b+t] = log sum_u exp(softmax_scale * q . k_u) (natural log).
 * An empty route gives O = 0 and lse = -inf.  route_ids == NULL computes
 * dense attention over all M tiles (route_len ignored).
 *
 * Q [H][N*b][d], K and V [H][M*b][d] bf16; O [H][N*b][d] bf16 out;
 * lse [H][N*b] fp32 out (nullable).  softmax_scale <= 0 means 1/sqrt(d).
 * row_order [H*N] (nullable): the (h*N + i) rows in the order the CTAs take
 * them, e.g. from velox_route_schedule; it must be a permutation of
 * 0 .. H*N-1 (an entry outside that range is skipped and flags
 * VELOX_DEV_BAD_ROW_ORDER).  The order changes no result.
 * d == b_tok == 128, M <= VELOX_MAX_BLOCKS, R_max <= VELOX_MAX_ROUTE when
 * routed.  A route id outside [0, M) or repeated within its row is skipped
 * (VELOX_DEV_BAD_ROUTE_ID / VELOX_DEV_DUP_ROUTE_ID); route_len outside
 * [0, R_max] zeroes the row (VELOX_DEV_ROUTE_LEN).  Q, K, V, O must be
 * 16-byte aligned.
 */
VELOX_API velox_status velox_block_sparse_attn(const velox_bf16 *Q, const velox_bf16 *K,
                                               const velox_bf16 *V,
                                               const int32_t *route_ids,
                                               const int32_t *route_len,
                                               const int32_t *row_order, int R_max,
                                               int H, int N, int M, int d, int b_tok,
                                               float softmax_scale, velox_bf16 *O,
                                               float *lse, int32_t *dev_status,
                                               velox_stream_t stream);

/*
 * velox_two_phase_attn -- routed history attention and the current chunk's
 * own keys in one softmax.
 *
 * Defined by: digest, "Reproducibility" (the two-phase tile loop) and
 * "Core method" (Eq. 15); project page, "02 · Method", step 04.  Reading:
 * every query token of block i attends to the tokens of its routed history
 * tiles (as velox_block_sparse_attn) and to all N_cur*b_tok tokens of the
 * current chunk, with one normaliser over both phases:
 *   O = sum over u in (routed history tokens) U (current tokens) of
 *       softmax_u(softmax_scale * q . k_u) v_u,   lse = log sum exp(...).
 *
 * K_cur, V_cur [H][N_cur*b][d] bf16 (16-byte aligned), N_cur > 0; all other
 * arguments, layouts, limits and device errors as velox_block_sparse_attn
 * (route_ids == NULL: all M history tiles).
 */
VELOX_API velox_status velox_two_phase_attn(const velox_bf16 *Q, const velox_bf16 *K,
                                            const velox_bf16 *V, const int32_t *route_ids,
                                            const int32_t *route_len,
                                            const int32_t *row_order, int R_max,
                                            const velox_bf16 *K_cur, const velox_bf16 *V_cur,
                                            int N_cur, int H, int N, int M, int d, int b_tok,
                                            float softmax_scale, velox_bf16 *O, float *lse,
                                            int32_t *dev_status, velox_stream_t stream);

/* A pinhole camera in latent-token units: pixel (u, v) at depth z is the
 * camera-frame point ((u - cx) / fx * z, (v - cy) / fy * z, z); the world
 * point is C + R x (R: world-from-camera rotation, row-major). */
typedef struct {
  float fx, fy, cx, cy;
  float R[9];
  float C[3];
} velox_camera;

/* A frustum slab: token rectangle [u0, u1) x [v0, v1) of camera `cam` and
 * the depth interval [zlo, zhi]; `valid` = 0 marks a block without reliable
 * geometry. */
typedef struct {
  float u0, u1, v0, v1, zlo, zhi;
  int32_t cam;
  int32_t valid;
} velox_slab;

/*
 * velox_slab_overlap -- g[i][r], the world-space overlap of query slab i and
 * history slab r.
 *
 * Defined by: project page, "02 · Method", glossary entry for g (overlap, IoU,
 * of the slabs in world space); digest, "Prerequisites" (frustum slab, OBB
 * overlap) and "Method steps", step three (Eq. 7).  Each slab is the
 * camera-facing oriented box with the camera's axes, centred on the ray
 * through the rectangle centre at the mid depth zm, half extents
 * (u1-u0)/(2 fx) zm, (v1-v0)/(2 fy) zm, (zhi-zlo)/2.  The intersection is
 * counted on the grid^3 cell centres of the query box:
 *   g = inter / (vol_i + vol_r - inter),  inter = vol_i * inside / grid^3;
 * an invalid history slab gives 0.
 *
 * cams [n_cams], q_slabs [N], h_slabs [M] (device), g [N][M] fp32 out.
 * 1 <= grid <= 32, N <= 65535 (VELOX_ERR_UNSUPPORTED otherwise).  A slab whose camera index is out of range gives 0 and
 * flags VELOX_DEV_BAD_CAMERA.
 */
VELOX_API velox_status velox_slab_overlap(const velox_camera *cams, int n_cams,
                                          const velox_slab *q_slabs, int N,
                                          const velox_slab *h_slabs, int M, int grid,
                                          float *g, int32_t *dev_status,
                                          velox_stream_t stream);

/*
 * velox_coverage -- rho[i], the fraction of query block i's tokens whose
 * warped depth falls inside a valid past slab, and covered[i] = rho >= eta.
 *
 * Defined by: digest, "Method steps", step three (Eq. 8: coverage and the
 * eta_cov = 0.9 threshold); onedev.kr summary, "How it differs" (a token is
 * covered when its multiwarp depth falls inside a valid past slab).
 * A token (u, v, z) of query block i (camera q_slabs[i].cam) is back-projected
 * and projected into each valid history slab's camera; it is covered when it
 * lands in the slab's rectangle at a depth in [zlo, zhi].  z <= 0 (a hole) is
 * never covered.
 *
 * q_uvz [N][b][3] fp32 (u, v, z per token), 1 <= b <= 128, N <= 2^29 (four
 * CTAs per query block); rho [N] fp32, covered [N] uint8 out.
 */
VELOX_API velox_status velox_coverage(const velox_camera *cams, int n_cams,
                                      const velox_slab *q_slabs, const float *q_uvz, int N,
                                      int b, const velox_slab *h_slabs, int M, float eta,
                                      float *rho, uint8_t *covered, int32_t *dev_status,
                                      velox_stream_t stream);

/*
 * velox_route_audit -- the geometry-model consistency audit, as six integer
 * counts per (head, query block) row.
 *
 * Defined by: project page, "03 · Results", "Geometry and the model agree"
 * (R_geo: positive-overlap blocks in the model's own top-50; fusion at
 * lambda = 2 raising the top-80 recall of positive-overlap blocks while
 * changing few selected blocks); digest, results table, row
 * "geometry-model importance consistency audit" (R_geo and the top-50
 * agreement R_50 against the random expectation 50/143); onedev.kr summary,
 * "Results".
 *
 * pos = {r : g[i][r] > tau}; top_K(x) = the K largest x_r, ties to the lower
 * id (all M when K >= M); fused = p (1 + lambda min(g / g_ref, 1) [g > tau])
 * in fp64 on every row.  counts[row][0..5] =
 *   |pos|, |pos & top_kgeo(p)|, |top_kgeo(g) & top_kgeo(p)|,
 *   |pos & top_kfuse(p)|, |pos & top_kfuse(fused)|,
 *   |top_kfuse(fused) - top_kfuse(p)|.
 * Pooled over rows: R_geo = sum c1 / sum c0, R_50 = sum c2 / (rows min(kgeo, M)),
 * top-kfuse recall = sum c3 (model) or sum c4 (fused) over sum c0,
 * changed = sum c5 / (rows min(kfuse, M)).
 *
 * p [H][N][M] fp32, g [N][M] fp32 (device), prm: host pointer (lambda, tau,
 * g_ref used), counts [H][N][6] int32 out.  M <= 4096 (VELOX_ERR_UNSUPPORTED
 * otherwise); k_geo, k_fuse >= 1.
 */
VELOX_API velox_status velox_route_audit(const float *p, const float *g, int H, int N, int M,
                                         const velox_route_params *prm, int k_geo, int k_fuse,
                                         int32_t *counts, velox_stream_t stream);

/*
 * velox_slab_table -- the frustum slab of every history block from depth.
 *
 * Defined by: digest, "Method steps", step one (Eq. 4-5: reliable depth
 * back-projected and bucketed by Gilbert block, 10/90 percentile depth
 * interval per block) and "Prerequisites" (a slab is a token rectangle plus
 * a depth interval); project page, "02 · Method", step 01.
 *
 * depth, conf [F][H s][W s] fp32 and mask [F][H s][W s] uint8 (conf and
 * mask nullable) hold global frames frame_base .. frame_base + F - 1, s x s
 * samples per token.  cell_of_rank [n_cells] is a token order (from
 * velox_gilbert_order or velox_thw_linear_order); block r covers ranks
 * r b_tok .. r b_tok + b_tok - 1.  For r = first_block + j, j < n_blocks:
 * slabs[j] = {u0, u1, v0, v1} = the bounding box [min x, max x + 1) x
 * [min y, max y + 1) of its cells, {zlo, zhi} = percentiles p_lo and p_hi
 * (linear interpolation between order statistics at (n - 1) p, fp64, rounded
 * to fp32) of its reliable samples (mask set, conf >= c_min, 0 < depth <
 * inf), cam = its global frame, valid = (n >= n_min); an invalid slab is all
 * zeros.  A block whose cells leave the lattice, straddle frames or lie
 * outside the given frames flags VELOX_DEV_BAD_CELL and is invalid.
 * token_uvz (nullable; only with s == 1) [n_blocks][b_tok][3]: the tokens of
 * each block in rank order as (x + 0.5, y + 0.5, depth), depth 0 where the
 * sample is not reliable -- the per-token input of velox_coverage when the
 * depth is a query frame's multiwarp depth.
 * Requires H W % b_tok == 0, 1 <= s, b_tok s^2 <= 16384.
 */
VELOX_API velox_status velox_slab_table(const float *depth, const float *conf,
                                        const uint8_t *mask, int F, int frame_base, int H, int W,
                                        int s, const int32_t *cell_of_rank, int n_cells,
                                        int b_tok, int first_block, int n_blocks, float c_min,
                                        int n_min, double p_lo, double p_hi, velox_slab *slabs,
                                        float *token_uvz, int32_t *dev_status,
                                        velox_stream_t stream);

/*
 * velox_multiwarp -- recency-priority multiwarp depth z^Q of target frames.
 *
 * Defined by: digest, "Method steps", step two (Eq. 6: first and last frame
 * depths of the K = 30 most recent reconstructed chunks forward-warped to the
 * target camera; each token takes the median of the newest frame that gives
 * it at least k_warp = 2 samples) and "Recency-priority multiwarp".
 *
 * src_depth [S][H s][W s] fp32 with cameras src_cam [S] (device), newest
 * first; tgt_cam [n_tgt] (device).  Every source sample (px, py) with depth
 * z > 0 sits at token coordinates ((px + 0.5) / s, (py + 0.5) / s); it is
 * back-projected with its camera and projected into the target camera; it
 * lands in target token (floor u', floor v') when its target depth is > 0
 * and 0 <= u' < W, 0 <= v' < H, with that depth as its value.
 * zq [n_tgt][H][W] fp32: the median (mean of the two middle values for an
 * even count, fp64 rounded to fp32) of the first source, newest first, that
 * gives the token >= k_warp samples; 0 (a hole) if none does.  A camera index
 * out of range flags VELOX_DEV_BAD_CAMERA and that source (target) is
 * skipped (left 0).  ws: caller-owned device workspace of at least
 * velox_multiwarp_workspace_size bytes (the per-source medians), else
 * VELOX_ERR_WORKSPACE.  Requires H W s^2 <= 32768 and H W <= 8192.
 */
VELOX_API velox_status velox_multiwarp(const velox_camera *cams, int n_cams,
                                       const float *src_depth, const int32_t *src_cam, int S,
                                       const int32_t *tgt_cam, int n_tgt, int H, int W, int s,
                                       int k_warp, float *zq, void *ws, size_t ws_bytes,
                                       int32_t *dev_status, velox_stream_t stream);

/* Bytes of workspace velox_multiwarp needs: 4 S n_tgt H W. */
VELOX_API velox_status velox_multiwarp_workspace_size(int S, int n_tgt, int H, int W,
                                                      size_t *bytes);

/*
 * velox_wait_selftest -- drive the library's bounded waits to their limit.
 *
 * The pages have no counterpart: this is the library's failure-detection
 * check.  Every kernel that waits on an mbarrier bounds the wait by the
 * device clock; a wait that gives up sets a CTA-wide abort flag, which ends
 * the CTA's other waits too, and the error is reported through dev_status
 * instead of a trap.  This call runs that code on one CTA of two warps:
 * thread 0 waits on a barrier that nothing completes, with a limit of
 * limit_us microseconds; the 32 threads of the second warp wait on another
 * such barrier with a limit ten times longer, which only the abort flag can
 * end at about limit_us.  Each warp that gives up OR-s VELOX_DEV_WAIT_TIMEOUT
 * into *dev_status.  elapsed_ns (device, nullable) [2] int64: how long thread
 * 0 and the second warp waited, in ns.  Nothing faults or traps and the
 * context stays usable.  1 <= limit_us <= 2,000,000, else
 * VELOX_ERR_INVALID_ARG.
 */
VELOX_API velox_status velox_wait_selftest(int limit_us, int32_t *dev_status,
                                           int64_t *elapsed_ns, velox_stream_t stream);

/*
 * velox_clock_probe -- sample the SM clock against the global timer.
 *
 * The pages have no counterpart: this is a measurement aid.  One CTA of one
 * warp; its thread 0 writes n pairs {clock64(), %globaltimer ns} to samples
 * (device, [n][2] int64), pausing about pause_ns nanoseconds between pairs.
 * Launched on its own stream beside another kernel, the ratio of successive
 * differences (cycles per ns) is the SM clock in GHz while that kernel runs
 * (the power limiter can hold it far below the clock the driver reports).
 * 1 <= n <= 1,000,000 and pause_ns <= 1,000,000, else VELOX_ERR_INVALID_ARG.
 */
VELOX_API velox_status velox_clock_probe(int64_t *samples, int n, int pause_ns,
                                         velox_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* VELOX_H_ */
