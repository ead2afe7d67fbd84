// Per-head block importance p_{i,r} = softmax_r(scale * qbar_i . kbar_r).
//
// Digest of arXiv 2610.22311, "Method steps", step four (Eq. 9); onedev.kr
// summary, "How it differs": each layer's block importance is the softmax of
// the mean-query / mean-key inner product.
//
// Three launches:
//   pool_kernel          query blocks: fp32 means qbar [H][N][d] into the
//                        workspace.  One warp per 128 x 128 bf16 block,
//                        16-byte non-caching loads, 16 in flight per lane.
//   pool_logits_kernel   streams K once (the HBM-bound part: 2.96 GB at the
//                        chunk-48 shape).  A CTA takes a contiguous range of
//                        one head's key blocks with that head's qbar in
//                        shared memory; each warp pools one block and its two
//                        half-warps dot the mean with half of the query rows
//                        each, while the warp's loads of its next block are
//                        in flight; logits are staged in shared memory and
//                        written into p row-contiguously.  No key means touch
//                        memory.
//   softmax_row_kernel   per (head, query block) row, one warp with the row
//                        in registers: max, exponentials and their sum,
//                        normalise, in place (softmax_kernel, a CTA per row
//                        with an online max/sum merge, for rows that do not
//                        fit).
// When N > kFusedMaxN the key means go through the workspace instead
// (pool_kernel on K, then logits_kernel).
#include "common.cuh"

namespace velox {
namespace {

constexpr int D = VELOX_HEAD_DIM;
constexpr int BT = VELOX_BLOCK_TOK;

__device__ __forceinline__ uint4 ld_stream(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void acc8(float (&a)[8], const uint4 &v) {
  a[0] += bf16_lo(v.x); a[1] += bf16_hi(v.x);
  a[2] += bf16_lo(v.y); a[3] += bf16_hi(v.y);
  a[4] += bf16_lo(v.z); a[5] += bf16_hi(v.z);
  a[6] += bf16_lo(v.w); a[7] += bf16_hi(v.w);
}

// Unit u < n_q: block u of Q (means to qbar); else block u - n_q of K (to kbar).
// Rows of a block are 256 bytes = 16 lanes x 16 bytes: lanes 0-15 take even
// rows, lanes 16-31 odd rows; each lane sums 8 channels over 64 rows, 16
// loads in flight at a time (the occupancy floor of one CTA leaves the
// compiler the registers for all 16; a chunk-48 launch has under two CTAs per
// SM anyway).
__global__ void __launch_bounds__(256, 1) pool_kernel(const uint16_t *__restrict__ Q,
                                                   const uint16_t *__restrict__ K, int n_q,
                                                   int n_units, float *__restrict__ qbar,
                                                   float *__restrict__ kbar) {
  const int lane = threadIdx.x & 31;
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int n_warps = (gridDim.x * blockDim.x) >> 5;
  const int col = (lane & 15) * 8;
  const int row0 = lane >> 4;
  for (int u = warp; u < n_units; u += n_warps) {
    const uint16_t *src;
    float *dst;
    if (u < n_q) {
      src = Q + (size_t)u * BT * D;
      dst = qbar + (size_t)u * D;
    } else {
      src = K + (size_t)(u - n_q) * BT * D;
      dst = kbar + (size_t)(u - n_q) * D;
    }
    float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    const uint16_t *p = src + row0 * D + col;
#pragma unroll 1
    for (int r = 0; r < BT / 2; r += 16) {
      uint4 v[16];
#pragma unroll
      for (int k = 0; k < 16; ++k) v[k] = ld_stream(p + (size_t)(r + k) * 2 * D);
#pragma unroll
      for (int k = 0; k < 16; ++k) acc8(a, v[k]);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) a[k] += __shfl_xor_sync(0xffffffffu, a[k], 16);
    if (lane < 16) {
      const float inv = 1.0f / BT;
      float4 lo = make_float4(a[0] * inv, a[1] * inv, a[2] * inv, a[3] * inv);
      float4 hi = make_float4(a[4] * inv, a[5] * inv, a[6] * inv, a[7] * inv);
      reinterpret_cast<float4 *>(dst + col)[0] = lo;
      reinterpret_cast<float4 *>(dst + col)[1] = hi;
    }
  }
}

// Logit tile: 64 history blocks per CTA, query rows 16 at a time.  The key
// means are stored transposed (channel-major) so that thread tx reads the
// 4 blocks 4*tx .. 4*tx+3 of one channel as a single float4; thread ty owns
// one query row of the current group.
constexpr int LG_R = 64;   // history blocks per CTA
constexpr int LG_Q = 16;   // query rows per pass

__global__ void __launch_bounds__(256) logits_kernel(const float *__restrict__ qbar,
                                                     const float *__restrict__ kbar, int N,
                                                     int M, float scale, float *__restrict__ p) {
  __shared__ __align__(16) float ks[D][LG_R + 4];
  __shared__ float qs[LG_Q][D + 4];
  const int h = blockIdx.y;
  const int r0 = blockIdx.x * LG_R;
  const int tid = threadIdx.x;
  const float *kb = kbar + ((size_t)h * M + r0) * D;
  for (int e = tid; e < LG_R * D / 4; e += blockDim.x) {
    int r = e / (D / 4), c = (e % (D / 4)) * 4;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (r0 + r < M) v = *reinterpret_cast<const float4 *>(kb + (size_t)r * D + c);
    ks[c][r] = v.x; ks[c + 1][r] = v.y; ks[c + 2][r] = v.z; ks[c + 3][r] = v.w;
  }
  const int ty = tid >> 4, tx = tid & 15;
  for (int i0 = 0; i0 < N; i0 += LG_Q) {
    __syncthreads();
    for (int e = tid; e < LG_Q * D / 4; e += blockDim.x) {
      int r = e / (D / 4), c = (e % (D / 4)) * 4;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      if (i0 + r < N)
        v = *reinterpret_cast<const float4 *>(qbar + ((size_t)h * N + i0 + r) * D + c);
      qs[r][c] = v.x; qs[r][c + 1] = v.y; qs[r][c + 2] = v.z; qs[r][c + 3] = v.w;
    }
    __syncthreads();
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int c = 0; c < D; ++c) {
      const float q = qs[ty][c];
      const float4 k4 = *reinterpret_cast<const float4 *>(&ks[c][4 * tx]);
      acc.x = fmaf(q, k4.x, acc.x);
      acc.y = fmaf(q, k4.y, acc.y);
      acc.z = fmaf(q, k4.z, acc.z);
      acc.w = fmaf(q, k4.w, acc.w);
    }
    const int i = i0 + ty;
    if (i < N) {
      float *dst = p + ((size_t)h * N + i) * M + r0 + 4 * tx;
      const float v[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (r0 + 4 * tx + k < M) dst[k] = scale * v[k];
    }
  }
}

// Fused K pooling + logits.  Grid-stride over chunks of 8 * per_warp key
// blocks of one head (chunk c: head c / cpr, blocks (c % cpr) * 8 * per_warp
// ..), 256 threads, grid sized to the resident capacity (two CTAs per SM:
// the registers of 16 loads in flight per lane plus the dot products);
// per_warp is the count whose busiest CTA streams the fewest blocks.
// Warp w of a CTA streams the per_warp consecutive key blocks r0 + w per_warp
// .. with no block-level barrier after the qbar load.  After the half-warp
// exchange both halves hold the 8 channel sums of lane (l & 15); half-warp 0
// computes the logits of query rows 0, 2, 4, ... and half-warp 1 of rows
// 1, 3, 5, ..., each as 8 products plus a 16-lane shuffle reduction, staged
// in the warp's own [N][8] shared-memory slice and written out row by row
// (8 consecutive logits = 32 bytes per row) once the warp's blocks are done.
// The warp's load stream does not stop for those products: the first 16
// loads of block k are issued before the products of block k - 1, which run
// while they are in flight.  Each sum and each product is formed in the same
// order as without the overlap.
constexpr int kFusedMaxN = 96;
constexpr int kFusedWarps = 8;
constexpr int kFusedPerWarp = 8;  // most key blocks per warp (the staging width)

__global__ void __launch_bounds__(kFusedWarps * 32) pool_logits_kernel(const uint16_t *__restrict__ K,
                                                          const float *__restrict__ qbar, int H,
                                                          int N, int M, float scale,
                                                          int per_warp, float *__restrict__ p) {
  extern __shared__ float4 fsm[];
  float *qs = reinterpret_cast<float *>(fsm);  // [N][D] means of the chunk's head
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float *lg = qs + N * D + warp * N * kFusedPerWarp;  // this warp's [N][8] logits
  const int col = (lane & 15) * 8;
  const int row0 = lane >> 4;
  const float cs = scale * (1.0f / BT);  // logit = scale * qbar . (sum / b)
  const int per_cta = kFusedWarps * per_warp;  // key blocks per chunk (per_warp <= 8)
  const int cpr = (M + per_cta - 1) / per_cta;
  for (int c = blockIdx.x; c < H * cpr; c += gridDim.x) {
  const int h = c / cpr;
  __syncthreads();  // every warp is done with the previous chunk's qbar
  for (int e = threadIdx.x; e < N * D / 4; e += blockDim.x)
    fsm[e] = reinterpret_cast<const float4 *>(qbar + (size_t)h * N * D)[e];
  __syncthreads();
  const int rw = (c - h * cpr) * per_cta + warp * per_warp;  // first block of the warp
  const int nb = min(per_warp, M - rw);  // this warp's blocks (none past M)
  float sum[8];  // channel sums of the previous block (both half-warps)
  for (int k = 0; nb > 0 && k <= nb; ++k) {
    const bool more = k < nb;  // uniform across the warp
    const uint16_t *src = K + ((size_t)h * M + rw + (more ? k : 0)) * BT * D + row0 * D + col;
    uint4 v[16];
    if (more) {
#pragma unroll
      for (int q = 0; q < 16; ++q) v[q] = ld_stream(src + (size_t)q * 2 * D);
    }
    if (k > 0) {
      // logits of block k - 1; same trip count in both half-warps (the
      // shuffles span the whole warp)
      for (int ii = 0; ii < (N + 1) / 2; ++ii) {
        const int i = 2 * ii + row0;
        const int iq = i < N ? i : N - 1;  // odd N: half-warp 1 repeats a row, unused
        const float4 q0 = *reinterpret_cast<const float4 *>(qs + iq * D + col);
        const float4 q1 = *reinterpret_cast<const float4 *>(qs + iq * D + col + 4);
        float d = q0.x * sum[0];
        d = fmaf(q0.y, sum[1], d); d = fmaf(q0.z, sum[2], d); d = fmaf(q0.w, sum[3], d);
        d = fmaf(q1.x, sum[4], d); d = fmaf(q1.y, sum[5], d); d = fmaf(q1.z, sum[6], d);
        d = fmaf(q1.w, sum[7], d);
#pragma unroll
        for (int off = 8; off > 0; off >>= 1) d += __shfl_xor_sync(0xffffffffu, d, off);
        if ((lane & 15) == 0 && i < N) lg[i * kFusedPerWarp + k - 1] = d * cs;
      }
    }
    if (more) {
      float a[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
      for (int q = 0; q < 16; ++q) acc8(a, v[q]);
#pragma unroll 1
      for (int r = 16; r < BT / 2; r += 16) {
#pragma unroll
        for (int q = 0; q < 16; ++q) v[q] = ld_stream(src + (size_t)(r + q) * 2 * D);
#pragma unroll
        for (int q = 0; q < 16; ++q) acc8(a, v[q]);
      }
#pragma unroll
      for (int q = 0; q < 8; ++q) sum[q] = a[q] + __shfl_xor_sync(0xffffffffu, a[q], 16);
    }
  }
  __syncwarp();
  for (int e = lane; e < N * kFusedPerWarp; e += 32) {
    const int i = e / kFusedPerWarp, k = e - i * kFusedPerWarp;
    if (k < nb) p[((size_t)h * N + i) * M + rw + k] = lg[e];
  }
  __syncwarp();
  }
}

__device__ __forceinline__ void merge_ms(float &m, float &s, float m2, float s2) {
  float mm = fmaxf(m, m2);
  if (mm == -INFINITY) return;
  s = s * expf(m - mm) + s2 * expf(m2 - mm);
  m = mm;
}

// One CTA per (h, i) row of M logits, in place; for rows the one-warp kernel
// below cannot hold (M above 4096, not a multiple of 4, or p not 16-byte aligned).
__global__ void __launch_bounds__(256) softmax_kernel(float *__restrict__ p, int M) {
  __shared__ float sm[8], ss[8];
  float *row = p + (size_t)blockIdx.x * M;
  float m = -INFINITY, s = 0.f;
  for (int r = threadIdx.x; r < M; r += blockDim.x) {
    float x = row[r];
    if (x > m) {
      s = s * expf(m - x) + 1.0f;
      m = x;
    } else {
      s += expf(x - m);
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    float m2 = __shfl_xor_sync(0xffffffffu, m, off);
    float s2 = __shfl_xor_sync(0xffffffffu, s, off);
    merge_ms(m, s, m2, s2);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) { sm[warp] = m; ss[warp] = s; }
  __syncthreads();
  if (warp == 0) {
    int nw = blockDim.x >> 5;
    m = lane < nw ? sm[lane] : -INFINITY;
    s = lane < nw ? ss[lane] : 0.f;
    for (int off = 16; off > 0; off >>= 1) {
      float m2 = __shfl_xor_sync(0xffffffffu, m, off);
      float s2 = __shfl_xor_sync(0xffffffffu, s, off);
      merge_ms(m, s, m2, s2);
    }
    if (lane == 0) { sm[0] = m; ss[0] = s; }
  }
  __syncthreads();
  const float gm = sm[0], inv = 1.0f / ss[0];
  for (int r = threadIdx.x; r < M; r += blockDim.x) row[r] = expf(row[r] - gm) * inv;
}

// One warp per (head, query block) row with the whole row in registers:
// VMAX float4 per lane, so rows of up to 128 * VMAX logits (M a multiple of 4,
// rows 16-byte aligned).  The row is read once and written once; each logit
// takes one exponential.
template <int VMAX>
__global__ void __launch_bounds__(256) softmax_row_kernel(float *__restrict__ p, int M,
                                                         int rows) {
  const int wrow = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wrow >= rows) return;  // uniform across the warp
  float4 *row = reinterpret_cast<float4 *>(p + (size_t)wrow * M);
  const int n4 = M >> 2;
  float4 x[VMAX];
#pragma unroll
  for (int j = 0; j < VMAX; ++j) {
    const int c = lane + 32 * j;
    x[j] = c < n4 ? row[c] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
  }
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < VMAX; ++j) m = fmaxf(m, fmaxf(fmaxf(x[j].x, x[j].y), fmaxf(x[j].z, x[j].w)));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < VMAX; ++j) {
    x[j].x = expf(x[j].x - m);  // padding: exp(-inf) = 0
    x[j].y = expf(x[j].y - m);
    x[j].z = expf(x[j].z - m);
    x[j].w = expf(x[j].w - m);
    s += (x[j].x + x[j].y) + (x[j].z + x[j].w);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  const float inv = 1.0f / s;
#pragma unroll
  for (int j = 0; j < VMAX; ++j) {
    const int c = lane + 32 * j;
    if (c < n4)
      row[c] = make_float4(x[j].x * inv, x[j].y * inv, x[j].z * inv, x[j].w * inv);
  }
}

}  // namespace

size_t importance_workspace_bytes(int H, int N, int M) {
  size_t b = (size_t)H * ((size_t)N + (size_t)M) * D * sizeof(float);
  return (b + 255) & ~(size_t)255;
}

cudaError_t launch_importance(const uint16_t *Q, const uint16_t *K, int H, int N, int M,
                              float scale, float *p, void *ws, cudaStream_t stream) {
  float *qbar = static_cast<float *>(ws);
  float *kbar = qbar + (size_t)H * N * D;
  const bool fused = N <= kFusedMaxN;
  const int n_q = H * N;
  const int n_units = fused ? n_q : H * (N + M);
  int grid = (n_units + 7) / 8;
  if (grid > 148 * 8 * 4) grid = 148 * 8 * 4;
  pool_kernel<<<grid, 256, 0, stream>>>(Q, K, n_q, n_units, qbar, kbar);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (fused) {
    const size_t smem = (size_t)N * (D + kFusedWarps * kFusedPerWarp) * sizeof(float);
    if (smem > 48 * 1024) {
      e = cudaFuncSetAttribute(pool_logits_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e != cudaSuccess) return e;
    }
    // CTA slots: what the registers and shared memory let reside per SM
    int per_sm = 0;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pool_logits_kernel,
                                                      kFusedWarps * 32, smem);
    if (e != cudaSuccess) return e;
    per_sm = per_sm < 1 ? 1 : per_sm;
    int dev = 0, sms = 0;
    e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    // key blocks per warp: the count (1..8) whose busiest CTA streams the
    // fewest blocks, i.e. ceil(chunks / slots) * per_warp smallest, the larger
    // count on ties (with 2 CTAs on each of 148 SMs and 2256 key blocks: 3 at
    // 40 heads, 5 at 20, 8 at 16, 5 at 10 and 5)
    const long long slots = (long long)sms * per_sm;
    int per_warp = kFusedPerWarp;
    long long best = -1;
    for (int pw = kFusedPerWarp; pw >= 1; --pw) {
      const long long ch = (long long)H * ((M + kFusedWarps * pw - 1) / (kFusedWarps * pw));
      const long long cost = (ch + slots - 1) / slots * pw;
      if (best < 0 || cost < best) {
        best = cost;
        per_warp = pw;
      }
    }
    const int chunks = H * ((M + kFusedWarps * per_warp - 1) / (kFusedWarps * per_warp));
    const int grid_f = chunks < slots ? chunks : (int)slots;
    pool_logits_kernel<<<grid_f, kFusedWarps * 32, smem, stream>>>(K, qbar, H, N, M, scale,
                                                                   per_warp, p);
  } else {
    dim3 lg((M + LG_R - 1) / LG_R, H);
    logits_kernel<<<lg, 256, 0, stream>>>(qbar, kbar, N, M, scale, p);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int rows = H * N;
  const int rgrid = (rows + 7) / 8;  // eight rows (warps) per CTA
  if ((M & 3) != 0 || (reinterpret_cast<uintptr_t>(p) & 15u) != 0 || M > 128 * 32) {
    softmax_kernel<<<rows, 256, 0, stream>>>(p, M);
  } else if (M <= 128 * 8) {
    softmax_row_kernel<8><<<rgrid, 256, 0, stream>>>(p, M, rows);
  } else if (M <= 128 * 18) {
    softmax_row_kernel<18><<<rgrid, 256, 0, stream>>>(p, M, rows);
  } else {
    softmax_row_kernel<32><<<rgrid, 256, 0, stream>>>(p, M, rows);
  }
  return cudaGetLastError();
}

}  // namespace velox
