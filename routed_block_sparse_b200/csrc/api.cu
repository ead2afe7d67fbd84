// C ABI of the velox library: argument validation and kernel dispatch.
//
// Every entry point checks its arguments on the host, returns a velox_status
// before launching anything when they are wrong, and otherwise enqueues its
// kernels on the caller's stream.  No entry point allocates device memory.
#include <cmath>
#include <cstddef>

#include "common.cuh"

namespace velox {
cudaError_t launch_gilbert(int T, int H, int W, int n_chunks, int b, int q_chunk,
                           int cache_first, int n_cache, int32_t *rank_of_cell,
                           int32_t *cell_of_rank, int32_t *block_of_cell, int32_t *nbr_ids,
                           int32_t *nbr_cnt, int S_max, int thw, int32_t *dev_status,
                           cudaStream_t stream);
size_t importance_workspace_bytes(int H, int N, int M);
cudaError_t launch_importance(const uint16_t *Q, const uint16_t *K, int H, int N, int M,
                              float scale, float *p, void *ws, cudaStream_t stream);
size_t route_workspace_bytes(int H, int N, int M);
cudaError_t launch_route(const float *p, const float *g, const uint8_t *covered,
                         const velox_route_params *prm, int prev_begin, int prev_count,
                         const int32_t *nbr_ids, const int32_t *nbr_cnt, int S_max,
                         const int32_t *ref_ids, int n_ref, int H, int N, int M,
                         int32_t *route_ids, int32_t *route_len, int32_t *route_nbudget,
                         int R_max, void *ws, int32_t *dev_status, cudaStream_t stream);
cudaError_t launch_schedule(const int32_t *route_len, int rows, int R_max, int32_t *row_order,
                            cudaStream_t stream);
cudaError_t launch_attn(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const int32_t *route_ids, const int32_t *route_len,
                        const int32_t *row_order, int R_max, const uint16_t *K_cur,
                        const uint16_t *V_cur, int N_cur, int H, int N, int M,
                        float softmax_scale, uint16_t *O, float *lse, int32_t *dev_status,
                        cudaStream_t stream, bool *map_failed);
cudaError_t launch_slab_overlap(const velox_camera *cams, int n_cams, const velox_slab *qs, int N,
                                const velox_slab *hs, int M, int G, float *g,
                                int32_t *dev_status, cudaStream_t stream);
cudaError_t launch_coverage(const velox_camera *cams, int n_cams, const velox_slab *qs,
                            const float *q_uvz, int N, int b, const velox_slab *hs, int M,
                            float eta, float *rho, uint8_t *covered, int32_t *dev_status,
                            cudaStream_t stream);
int audit_max_blocks();
int multiwarp_max_samples();
int multiwarp_max_tokens();
size_t multiwarp_ws_bytes(int S, int n_tgt, int H, int W);
int slab_table_max_samples();
cudaError_t launch_slab_table(const float *depth, const float *conf, const uint8_t *mask, int F,
                              int frame_base, int H, int W, int s, const int32_t *cell_of_rank,
                              int n_cells, int b, int first_block, int n_blocks, float c_min,
                              int n_min, double p_lo, double p_hi, velox_slab *slabs,
                              float *token_uvz, int32_t *dev_status, cudaStream_t stream);
cudaError_t launch_multiwarp(const velox_camera *cams, int n_cams, const float *src_depth,
                             const int32_t *src_cam, int S, const int32_t *tgt_cam, int n_tgt,
                             int H, int W, int s, int k_warp, float *zq, void *ws,
                             int32_t *dev_status, cudaStream_t stream);
cudaError_t launch_audit(const float *p, const float *g, int H, int N, int M, double lam,
                         double tau, double g_ref, int k_geo, int k_fuse, int32_t *counts,
                         cudaStream_t stream);
cudaError_t launch_clock_probe(int64_t *samples, int n, uint32_t pause_ns, cudaStream_t stream);
cudaError_t launch_wait_selftest(uint64_t limit_ns, int32_t *dev_status, int64_t *elapsed_ns,
                                 cudaStream_t stream);
}  // namespace velox

namespace {

constexpr long long kInt32Max = 2147483647LL;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

velox_status from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return VELOX_OK;
  cudaGetLastError();  // clear a sticky launch-configuration error
  return VELOX_ERR_CUDA;
}

// The device must be a Blackwell data-centre part (compute capability 10.x).
velox_status check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return VELOX_ERR_DEVICE;
  }
  static thread_local int cached_dev = -1, cached_major = 0;
  if (cached_dev != dev) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
      cudaGetLastError();
      return VELOX_ERR_DEVICE;
    }
    cached_dev = dev;
    cached_major = major;
  }
  return cached_major == 10 ? VELOX_OK : VELOX_ERR_DEVICE;
}

size_t workspace_bytes(int H, int N, int M) {
  size_t a = velox::importance_workspace_bytes(H, N, M);
  size_t b = velox::route_workspace_bytes(H, N, M);
  return a > b ? a : b;
}

}  // namespace

extern "C" {

const char *velox_status_string(velox_status s) {
  switch (s) {
    case VELOX_OK: return "ok";
    case VELOX_ERR_INVALID_ARG: return "invalid argument";
    case VELOX_ERR_UNSUPPORTED: return "unsupported size or shape";
    case VELOX_ERR_WORKSPACE: return "workspace missing or too small";
    case VELOX_ERR_CAPACITY: return "output capacity too small";
    case VELOX_ERR_DEVICE: return "no usable sm_100 device";
    case VELOX_ERR_TIMEOUT: return "bounded device wait gave up";
    case VELOX_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

int velox_abi_version(void) { return 104; }

}  // extern "C"

namespace {

velox_status order_common(int T, int H, int W, int n_chunks, int b_tok, int q_chunk,
                          int cache_first_block, int n_cache_blocks, int32_t *rank_of_cell,
                          int32_t *cell_of_rank, int32_t *block_of_cell, int32_t *nbr_ids,
                          int32_t *nbr_cnt, int S_max, int thw, int32_t *dev_status,
                          velox_stream_t stream) {
  if (T <= 0 || H <= 0 || W <= 0 || n_chunks <= 0 || b_tok <= 0) return VELOX_ERR_INVALID_ARG;
  if (velox::product_exceeds({n_chunks, T, H, W}, kInt32Max)) return VELOX_ERR_UNSUPPORTED;
  if (!thw && (W < H || (W % 2 == 1 && H % 2 == 0))) return VELOX_ERR_UNSUPPORTED;
  if (((long long)T * H * W) % b_tok != 0) return VELOX_ERR_UNSUPPORTED;
  if (b_tok > 1024) return VELOX_ERR_UNSUPPORTED;
  const bool want_nbr = nbr_ids != nullptr || nbr_cnt != nullptr;
  if (want_nbr) {
    if (q_chunk < 0 || q_chunk >= n_chunks) return VELOX_ERR_INVALID_ARG;
    const long long total_blocks = (long long)n_chunks * T * H * W / b_tok;
    if (cache_first_block < 0 || n_cache_blocks < 0 ||
        (long long)cache_first_block + n_cache_blocks > total_blocks)
      return VELOX_ERR_INVALID_ARG;
    if (S_max < 0 || (nbr_ids != nullptr && S_max == 0)) return VELOX_ERR_CAPACITY;
    if (dev_status == nullptr) return VELOX_ERR_INVALID_ARG;
  }
  if (!want_nbr && !rank_of_cell && !cell_of_rank && !block_of_cell) return VELOX_OK;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_gilbert(T, H, W, n_chunks, b_tok, q_chunk, cache_first_block,
                                         n_cache_blocks, rank_of_cell, cell_of_rank,
                                         block_of_cell, nbr_ids, nbr_cnt, S_max, thw, dev_status,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

}  // namespace

extern "C" {

velox_status velox_gilbert_order(int T, int H, int W, int n_chunks, int b_tok, int q_chunk,
                                 int cache_first_block, int n_cache_blocks,
                                 int32_t *rank_of_cell, int32_t *cell_of_rank,
                                 int32_t *block_of_cell, int32_t *nbr_ids, int32_t *nbr_cnt,
                                 int S_max, int32_t *dev_status, velox_stream_t stream) {
  return order_common(T, H, W, n_chunks, b_tok, q_chunk, cache_first_block, n_cache_blocks,
                      rank_of_cell, cell_of_rank, block_of_cell, nbr_ids, nbr_cnt, S_max, 0,
                      dev_status, stream);
}

velox_status velox_thw_linear_order(int T, int H, int W, int n_chunks, int b_tok, int q_chunk,
                                    int cache_first_block, int n_cache_blocks,
                                    int32_t *rank_of_cell, int32_t *cell_of_rank,
                                    int32_t *block_of_cell, int32_t *nbr_ids, int32_t *nbr_cnt,
                                    int S_max, int32_t *dev_status, velox_stream_t stream) {
  return order_common(T, H, W, n_chunks, b_tok, q_chunk, cache_first_block, n_cache_blocks,
                      rank_of_cell, cell_of_rank, block_of_cell, nbr_ids, nbr_cnt, S_max, 1,
                      dev_status, stream);
}

velox_status velox_workspace_size(int H, int N, int M, int d, size_t *bytes) {
  if (bytes == nullptr || H <= 0 || N <= 0 || M <= 0) return VELOX_ERR_INVALID_ARG;
  if (d != VELOX_HEAD_DIM) return VELOX_ERR_UNSUPPORTED;
  if (M > VELOX_MAX_BLOCKS) return VELOX_ERR_UNSUPPORTED;
  *bytes = workspace_bytes(H, N, M);
  return VELOX_OK;
}

velox_status velox_block_importance(const velox_bf16 *Q, const velox_bf16 *K, int H, int N,
                                    int M, int d, int b_tok, float scale, float *p, void *ws,
                                    size_t ws_bytes, velox_stream_t stream) {
  if (!Q || !K || !p || H <= 0 || N <= 0 || M <= 0) return VELOX_ERR_INVALID_ARG;
  if (d != VELOX_HEAD_DIM || b_tok != VELOX_BLOCK_TOK) return VELOX_ERR_UNSUPPORTED;
  if (M > VELOX_MAX_BLOCKS || velox::product_exceeds({H, M, b_tok}, kInt32Max) ||
      velox::product_exceeds({H, N, b_tok}, kInt32Max))
    return VELOX_ERR_UNSUPPORTED;
  if (!std::isfinite(scale)) return VELOX_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(p)) return VELOX_ERR_INVALID_ARG;
  if (ws == nullptr || ws_bytes < velox::importance_workspace_bytes(H, N, M) || !aligned16(ws))
    return VELOX_ERR_WORKSPACE;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_importance(Q, K, H, N, M, scale, p, ws,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

velox_status velox_route_build(const float *p, const float *g, const uint8_t *covered,
                               const velox_route_params *prm, int prev_begin, int prev_count,
                               const int32_t *nbr_ids, const int32_t *nbr_cnt, int S_max,
                               const int32_t *ref_ids, int n_ref, int H, int N, int M,
                               int32_t *route_ids, int32_t *route_len, int32_t *route_nbudget,
                               int R_max, void *ws, size_t ws_bytes, int32_t *dev_status,
                               velox_stream_t stream) {
  if (!p || !g || !covered || !prm || !route_ids || !route_len || !route_nbudget || !dev_status)
    return VELOX_ERR_INVALID_ARG;
  if (H <= 0 || N <= 0 || M <= 0) return VELOX_ERR_INVALID_ARG;
  if (M > VELOX_MAX_BLOCKS) return VELOX_ERR_UNSUPPORTED;
  if ((long long)H * N > kInt32Max / 2) return VELOX_ERR_UNSUPPORTED;
  if (prev_begin < 0 || prev_count < 0 || (long long)prev_begin + prev_count > M)
    return VELOX_ERR_INVALID_ARG;
  if (prm->k_cov < 0 || prm->k_unc < 0) return VELOX_ERR_INVALID_ARG;
  if (prm->k_cov > VELOX_MAX_ROUTE || prm->k_unc > VELOX_MAX_ROUTE) return VELOX_ERR_UNSUPPORTED;
  if (!std::isfinite(prm->lambda) || !std::isfinite(prm->tau) || !std::isfinite(prm->g_ref) ||
      !(prm->g_ref > 0.f) || !(prm->lambda >= 0.f) || std::isnan(prm->theta_cov) ||
      std::isnan(prm->theta_unc))
    return VELOX_ERR_INVALID_ARG;
  const bool have_nbr = (nbr_ids != nullptr || nbr_cnt != nullptr) && S_max > 0;
  if (have_nbr && (nbr_ids == nullptr || nbr_cnt == nullptr)) return VELOX_ERR_INVALID_ARG;
  if (S_max < 0 || n_ref < 0) return VELOX_ERR_INVALID_ARG;
  if (n_ref > 0 && ref_ids == nullptr) return VELOX_ERR_INVALID_ARG;
  const int s_eff = have_nbr ? S_max : 0;
  long long kmax = prm->k_cov > prm->k_unc ? prm->k_cov : prm->k_unc;
  if (prev_count > kmax) kmax = prev_count;
  long long need = kmax + s_eff + n_ref;
  if (need > M) need = M;
  if (R_max < need || R_max <= 0) return VELOX_ERR_CAPACITY;
  const size_t ws_need = velox::route_workspace_bytes(H, N, M);
  if (ws_need > 0 && (ws == nullptr || ws_bytes < ws_need)) return VELOX_ERR_WORKSPACE;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_route(p, g, covered, prm, prev_begin, prev_count,
                                       have_nbr ? nbr_ids : nullptr, have_nbr ? nbr_cnt : nullptr,
                                       s_eff, ref_ids, n_ref, H, N, M, route_ids, route_len,
                                       route_nbudget, R_max, ws, dev_status,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

velox_status velox_route_schedule(const int32_t *route_len, int rows, int R_max,
                                  int32_t *row_order, velox_stream_t stream) {
  if (!route_len || !row_order || rows <= 0 || R_max <= 0) return VELOX_ERR_INVALID_ARG;
  if (R_max > VELOX_MAX_ROUTE) return VELOX_ERR_UNSUPPORTED;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_schedule(route_len, rows, R_max, row_order,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"

namespace {

velox_status attn_common(const velox_bf16 *Q, const velox_bf16 *K, const velox_bf16 *V,
                         const int32_t *route_ids, const int32_t *route_len,
                         const int32_t *row_order, int R_max, const velox_bf16 *K_cur,
                         const velox_bf16 *V_cur, int N_cur, int H, int N, int M, int d,
                         int b_tok, float softmax_scale, velox_bf16 *O, float *lse,
                         int32_t *dev_status, velox_stream_t stream) {
  if (!Q || !K || !V || !O || H <= 0 || N <= 0 || M <= 0) return VELOX_ERR_INVALID_ARG;
  if (d != VELOX_HEAD_DIM || b_tok != VELOX_BLOCK_TOK) return VELOX_ERR_UNSUPPORTED;
  if (M > VELOX_MAX_BLOCKS || (long long)M * b_tok > kInt32Max ||
      (long long)N * b_tok > kInt32Max || (long long)H * N > kInt32Max)
    return VELOX_ERR_UNSUPPORTED;
  if (row_order != nullptr && dev_status == nullptr) return VELOX_ERR_INVALID_ARG;
  if (route_ids != nullptr) {
    if (route_len == nullptr || dev_status == nullptr) return VELOX_ERR_INVALID_ARG;
    if (R_max <= 0) return VELOX_ERR_INVALID_ARG;
    if (R_max > VELOX_MAX_ROUTE) return VELOX_ERR_UNSUPPORTED;
  }
  if (N_cur < 0) return VELOX_ERR_INVALID_ARG;
  if (N_cur > 0) {
    if (!K_cur || !V_cur) return VELOX_ERR_INVALID_ARG;
    if ((long long)N_cur * b_tok > kInt32Max) return VELOX_ERR_UNSUPPORTED;
    if (!aligned16(K_cur) || !aligned16(V_cur)) return VELOX_ERR_INVALID_ARG;
  }
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return VELOX_ERR_INVALID_ARG;
  if (std::isnan(softmax_scale) || std::isinf(softmax_scale)) return VELOX_ERR_INVALID_ARG;
  const float scale = softmax_scale > 0.f ? softmax_scale : 1.0f / std::sqrt((float)d);
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  bool map_failed = false;
  cudaError_t e = velox::launch_attn(Q, K, V, route_ids, route_len, row_order, R_max,
                                     N_cur > 0 ? K_cur : nullptr, N_cur > 0 ? V_cur : nullptr,
                                     N_cur, H, N, M, scale, O, lse, dev_status,
                                     reinterpret_cast<cudaStream_t>(stream), &map_failed);
  if (map_failed) return VELOX_ERR_CUDA;
  return from_cuda(e);
}

}  // namespace

extern "C" {

velox_status velox_block_sparse_attn(const velox_bf16 *Q, const velox_bf16 *K,
                                     const velox_bf16 *V, const int32_t *route_ids,
                                     const int32_t *route_len, const int32_t *row_order,
                                     int R_max, int H, int N, int M, int d, int b_tok,
                                     float softmax_scale, velox_bf16 *O, float *lse,
                                     int32_t *dev_status, velox_stream_t stream) {
  return attn_common(Q, K, V, route_ids, route_len, row_order, R_max, nullptr, nullptr, 0, H, N,
                     M, d, b_tok, softmax_scale, O, lse, dev_status, stream);
}

velox_status velox_two_phase_attn(const velox_bf16 *Q, const velox_bf16 *K, const velox_bf16 *V,
                                  const int32_t *route_ids, const int32_t *route_len,
                                  const int32_t *row_order, int R_max, const velox_bf16 *K_cur,
                                  const velox_bf16 *V_cur, int N_cur, int H, int N, int M, int d,
                                  int b_tok, float softmax_scale, velox_bf16 *O, float *lse,
                                  int32_t *dev_status, velox_stream_t stream) {
  if (N_cur <= 0 || !K_cur || !V_cur) return VELOX_ERR_INVALID_ARG;
  return attn_common(Q, K, V, route_ids, route_len, row_order, R_max, K_cur, V_cur, N_cur, H, N,
                     M, d, b_tok, softmax_scale, O, lse, dev_status, stream);
}

velox_status velox_slab_overlap(const velox_camera *cams, int n_cams, const velox_slab *q_slabs,
                                int N, const velox_slab *h_slabs, int M, int grid, float *g,
                                int32_t *dev_status, velox_stream_t stream) {
  if (!cams || !q_slabs || !h_slabs || !g || !dev_status) return VELOX_ERR_INVALID_ARG;
  if (n_cams <= 0 || N <= 0 || M <= 0 || grid < 1) return VELOX_ERR_INVALID_ARG;
  if (grid > 32 || N > 65535 || (long long)N * M > kInt32Max) return VELOX_ERR_UNSUPPORTED;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_slab_overlap(cams, n_cams, q_slabs, N, h_slabs, M, grid, g,
                                              dev_status, reinterpret_cast<cudaStream_t>(stream)));
}

velox_status velox_coverage(const velox_camera *cams, int n_cams, const velox_slab *q_slabs,
                            const float *q_uvz, int N, int b, const velox_slab *h_slabs, int M,
                            float eta, float *rho, uint8_t *covered, int32_t *dev_status,
                            velox_stream_t stream) {
  if (!cams || !q_slabs || !q_uvz || !h_slabs || !rho || !covered || !dev_status)
    return VELOX_ERR_INVALID_ARG;
  if (n_cams <= 0 || N <= 0 || M <= 0 || b <= 0 || std::isnan(eta)) return VELOX_ERR_INVALID_ARG;
  if (b > 128 || N > kInt32Max / 4) return VELOX_ERR_UNSUPPORTED;  // 4 CTAs per query block
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_coverage(cams, n_cams, q_slabs, q_uvz, N, b, h_slabs, M, eta, rho,
                                          covered, dev_status,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

velox_status velox_route_audit(const float *p, const float *g, int H, int N, int M,
                              const velox_route_params *prm, int k_geo, int k_fuse,
                              int32_t *counts, velox_stream_t stream) {
  if (!p || !g || !prm || !counts || H <= 0 || N <= 0 || M <= 0) return VELOX_ERR_INVALID_ARG;
  if (k_geo < 1 || k_fuse < 1) return VELOX_ERR_INVALID_ARG;
  if (!std::isfinite(prm->lambda) || !std::isfinite(prm->tau) || !std::isfinite(prm->g_ref) ||
      !(prm->g_ref > 0.f) || !(prm->lambda >= 0.f))
    return VELOX_ERR_INVALID_ARG;
  if (M > velox::audit_max_blocks() || (long long)H * N > kInt32Max) return VELOX_ERR_UNSUPPORTED;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_audit(p, g, H, N, M, prm->lambda, prm->tau, prm->g_ref, k_geo,
                                       k_fuse, counts, reinterpret_cast<cudaStream_t>(stream)));
}

velox_status velox_slab_table(const float *depth, const float *conf, const uint8_t *mask, int F,
                             int frame_base, int H, int W, int s, const int32_t *cell_of_rank,
                             int n_cells, int b_tok, int first_block, int n_blocks, float c_min,
                             int n_min, double p_lo, double p_hi, velox_slab *slabs,
                             float *token_uvz, int32_t *dev_status, velox_stream_t stream) {
  if (!depth || !cell_of_rank || !slabs || !dev_status) return VELOX_ERR_INVALID_ARG;
  if (token_uvz && s != 1) return VELOX_ERR_UNSUPPORTED;
  if (F <= 0 || H <= 0 || W <= 0 || s <= 0 || b_tok <= 0 || n_blocks <= 0 || first_block < 0 ||
      n_cells <= 0 || n_min < 0)
    return VELOX_ERR_INVALID_ARG;
  if (!(p_lo >= 0.0 && p_lo <= 1.0 && p_hi >= 0.0 && p_hi <= 1.0) || std::isnan(c_min))
    return VELOX_ERR_INVALID_ARG;
  if ((long long)(first_block + (long long)n_blocks) * b_tok > n_cells) return VELOX_ERR_INVALID_ARG;
  if (((long long)H * W) % b_tok != 0) return VELOX_ERR_UNSUPPORTED;
  if (velox::product_exceeds({b_tok, s, s}, velox::slab_table_max_samples()))
    return VELOX_ERR_UNSUPPORTED;
  if (velox::product_exceeds({F, H, W, s, s}, kInt32Max) || n_blocks > kInt32Max / 2)
    return VELOX_ERR_UNSUPPORTED;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_slab_table(depth, conf, mask, F, frame_base, H, W, s,
                                            cell_of_rank, n_cells, b_tok, first_block, n_blocks,
                                            c_min, n_min, p_lo, p_hi, slabs, token_uvz, dev_status,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

velox_status velox_multiwarp_workspace_size(int S, int n_tgt, int H, int W, size_t *bytes) {
  if (!bytes || S <= 0 || n_tgt <= 0 || H <= 0 || W <= 0) return VELOX_ERR_INVALID_ARG;
  *bytes = velox::multiwarp_ws_bytes(S, n_tgt, H, W);
  return VELOX_OK;
}

velox_status velox_multiwarp(const velox_camera *cams, int n_cams, const float *src_depth,
                             const int32_t *src_cam, int S, const int32_t *tgt_cam, int n_tgt,
                             int H, int W, int s, int k_warp, float *zq, void *ws,
                             size_t ws_bytes, int32_t *dev_status, velox_stream_t stream) {
  if (!cams || !src_depth || !src_cam || !tgt_cam || !zq || !dev_status)
    return VELOX_ERR_INVALID_ARG;
  if (n_cams <= 0 || S <= 0 || n_tgt <= 0 || H <= 0 || W <= 0 || s <= 0 || k_warp < 1)
    return VELOX_ERR_INVALID_ARG;
  if (velox::product_exceeds({H, W, s, s}, velox::multiwarp_max_samples()) ||
      velox::product_exceeds({H, W}, velox::multiwarp_max_tokens()) || n_tgt > 65535 ||
      S > 65535)
    return VELOX_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < velox::multiwarp_ws_bytes(S, n_tgt, H, W)) return VELOX_ERR_WORKSPACE;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_multiwarp(cams, n_cams, src_depth, src_cam, S, tgt_cam, n_tgt, H,
                                           W, s, k_warp, zq, ws, dev_status,
                                           reinterpret_cast<cudaStream_t>(stream)));
}

velox_status velox_clock_probe(int64_t *samples, int n, int pause_ns, velox_stream_t stream) {
  if (!samples || n < 1 || n > 1000000 || pause_ns < 0 || pause_ns > 1000000)
    return VELOX_ERR_INVALID_ARG;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_clock_probe(samples, n, static_cast<uint32_t>(pause_ns),
                                             reinterpret_cast<cudaStream_t>(stream)));
}

velox_status velox_wait_selftest(int limit_us, int32_t *dev_status, int64_t *elapsed_ns,
                                 velox_stream_t stream) {
  if (!dev_status || limit_us < 1 || limit_us > 2000000) return VELOX_ERR_INVALID_ARG;
  velox_status st = check_device();
  if (st != VELOX_OK) return st;
  return from_cuda(velox::launch_wait_selftest(static_cast<uint64_t>(limit_us) * 1000u,
                                               dev_status, elapsed_ns,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
