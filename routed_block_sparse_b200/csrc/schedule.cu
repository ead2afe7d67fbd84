// velox_route_schedule: the launch order of the attention rows, longest
// route first.
//
// A launch-order hint only (the pages have no counterpart): CTAs of the
// attention kernel take rows in this order, so the long rows start early and
// the last wave is made of short ones.  Counting sort by length, descending,
// stable in the row index (rows of one head stay together within a length).
#include "common.cuh"

namespace velox {
namespace {

constexpr int kThreads = 1024;
constexpr int kKeepRows = 8192;  // rows whose bins stay in shared memory

__global__ void __launch_bounds__(kThreads) schedule_kernel(const int32_t *__restrict__ route_len,
                                                            int rows, int R_max,
                                                            int32_t *__restrict__ row_order) {
  extern __shared__ int bins[];  // R_max + 1 counters, bin k = length R_max - k
  __shared__ int s_warp[kThreads / 32];
  const int nb = R_max + 1;
  // the bin of every row, kept for the placement pass when it fits (one warp
  // walks the rows in order there, and a global load per step would set its
  // pace)
  int *row_bin = bins + nb;
  const bool keep = rows <= kKeepRows;
  for (int k = threadIdx.x; k < nb; k += kThreads) bins[k] = 0;
  __syncthreads();
  for (int r = threadIdx.x; r < rows; r += kThreads) {
    int L = route_len[r];
    L = (L < 0 || L > R_max) ? 0 : L;
    atomicAdd(&bins[R_max - L], 1);
    if (keep) row_bin[r] = R_max - L;
  }
  __syncthreads();
  // exclusive scan of the bins (thread t owns a contiguous run)
  const int per = (nb + kThreads - 1) / kThreads;
  const int lo = min(nb, (int)threadIdx.x * per), hi = min(nb, lo + per);
  int mine = 0;
  for (int k = lo; k < hi; ++k) mine += bins[k];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = mine;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += s_warp[w];
  int run = before + incl - mine;
  for (int k = lo; k < hi; ++k) {
    const int c = bins[k];
    bins[k] = run;
    run += c;
  }
  __syncthreads();
  // stable placement by one warp, 32 rows at a time
  if (warp == 0) {
    for (int base = 0; base < rows; base += 32) {
      const int r = base + lane;
      int bin = -1;
      if (r < rows) {
        if (keep) {
          bin = row_bin[r];
        } else {
          int L = route_len[r];
          L = (L < 0 || L > R_max) ? 0 : L;
          bin = R_max - L;
        }
      }
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      const int rank = __popc(peers & ((1u << lane) - 1u));
      int start = 0;
      if (r < rows) start = bins[bin];
      __syncwarp();
      if (r < rows) {
        row_order[start + rank] = r;
        if (rank == 0) bins[bin] = start + __popc(peers);
      }
      __syncwarp();
    }
  }
}

}  // namespace

cudaError_t launch_schedule(const int32_t *route_len, int rows, int R_max, int32_t *row_order,
                            cudaStream_t stream) {
  const size_t smem = ((size_t)(R_max + 1) + (rows <= kKeepRows ? (size_t)rows : 0)) * sizeof(int);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(schedule_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  schedule_kernel<<<1, kThreads, smem, stream>>>(route_len, rows, R_max, row_order);
  return cudaGetLastError();
}

}  // namespace velox
