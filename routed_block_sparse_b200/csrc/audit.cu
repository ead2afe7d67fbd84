// Geometry-model consistency audit: per-row counts behind R_geo, R_50 and
// the top-K recall of the positive-overlap blocks with and without fusion.
//
// Velox project page, "03 · Results", "Geometry and the model agree"; digest
// of arXiv 2610.22311, results table, row "geometry-model importance
// consistency audit"; onedev.kr summary, "Results".  Positive blocks are
// those with g > tau; a top-K is the K largest scores, ties to the lower id.
//
// One CTA per (head, query block) row.  The three scores of the row (p, g
// and the fused weight p (1 + lambda g^), fp64 with explicitly rounded
// operations) sit in shared memory; every block's rank under each score is
// counted directly (M <= 4096), so membership of each top-K is exact.  Six
// counts per row:
//   0 |pos|                     1 |pos & top_geo(p)|
//   2 |top_geo(g) & top_geo(p)| 3 |pos & top_fuse(p)|
//   4 |pos & top_fuse(fused)|   5 |top_fuse(fused) - top_fuse(p)|
#include "common.cuh"

namespace velox {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct AuditArgs {
  const float *p;  // [rows][M]
  const float *g;  // [N][M]
  int N, M;
  double lam, tau, g_ref;
  int k_geo, k_fuse;
  int32_t *counts;  // [rows][6]
};

// Number of blocks ahead of r: larger score, or equal score and lower id.
__device__ __forceinline__ int rank_of(const double *key, int M, int r) {
  const double x = key[r];
  int n = 0;
  for (int s = 0; s < M; ++s) {
    const double y = key[s];
    n += (y > x) || (y == x && s < r);
  }
  return n;
}

__global__ void __launch_bounds__(kThreads) audit_kernel(AuditArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int s_red[6][kWarps];
  const int M = a.M;
  double *kp = reinterpret_cast<double *>(smem_raw);
  double *kg = kp + M;
  double *kf = kg + M;
  const int row = blockIdx.x;
  const int i = row % a.N;
  const float *prow = a.p + (size_t)row * M;
  const float *grow = a.g + (size_t)i * M;
  for (int r = threadIdx.x; r < M; r += kThreads) {
    const double pv = static_cast<double>(prow[r]);
    const double gv = static_cast<double>(grow[r]);
    double gh = 0.0;
    if (gv > a.tau) {
      gh = __ddiv_rn(gv, a.g_ref);
      if (gh > 1.0) gh = 1.0;
    }
    const double w = __dmul_rn(pv, __dadd_rn(1.0, __dmul_rn(a.lam, gh)));
    kp[r] = __dadd_rn(pv, 0.0);  // -0 -> +0: zeros tie exactly
    kg[r] = __dadd_rn(gv, 0.0);
    kf[r] = __dadd_rn(w, 0.0);
  }
  __syncthreads();
  int c[6] = {0, 0, 0, 0, 0, 0};
  for (int r = threadIdx.x; r < M; r += kThreads) {
    const bool pos = kg[r] > a.tau;
    const int rp = rank_of(kp, M, r), rg = rank_of(kg, M, r), rf = rank_of(kf, M, r);
    const bool in_pg = rp < a.k_geo, in_pf = rp < a.k_fuse;
    const bool in_gg = rg < a.k_geo, in_ff = rf < a.k_fuse;
    c[0] += pos;
    c[1] += pos && in_pg;
    c[2] += in_gg && in_pg;
    c[3] += pos && in_pf;
    c[4] += pos && in_ff;
    c[5] += in_ff && !in_pf;
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int k = 0; k < 6; ++k) {
    int v = c[k];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) s_red[k][warp] = v;
  }
  __syncthreads();
  if (threadIdx.x < 6) {
    int t = 0;
    for (int w = 0; w < kWarps; ++w) t += s_red[threadIdx.x][w];
    a.counts[(size_t)row * 6 + threadIdx.x] = t;
  }
}

}  // namespace

int audit_max_blocks() { return 4096; }

cudaError_t launch_audit(const float *p, const float *g, int H, int N, int M, double lam,
                         double tau, double g_ref, int k_geo, int k_fuse, int32_t *counts,
                         cudaStream_t stream) {
  AuditArgs a;
  a.p = p;
  a.g = g;
  a.N = N;
  a.M = M;
  a.lam = lam;
  a.tau = tau;
  a.g_ref = g_ref;
  a.k_geo = k_geo;
  a.k_fuse = k_fuse;
  a.counts = counts;
  const size_t smem = 3 * sizeof(double) * (size_t)M;
  cudaError_t e = cudaFuncSetAttribute(audit_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  audit_kernel<<<H * N, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace velox
