// Slab-table build and recency-priority multiwarp: the history-side and
// query-side geometry that the slab overlap and the coverage consume.
//
// Digest of arXiv 2610.22311, "Method steps", steps one and two (Eq. 4-6),
// and "Prerequisites" (frustum slab); Velox project page, "02 · Method",
// steps 01-02; onedev.kr summary, "How it differs".
//
//   slab_table_kernel   one CTA per history block: the block's cells come
//                       from the token order (cell_of_rank), its rectangle is
//                       their bounding box, its depth interval the p_lo / p_hi
//                       percentiles (linear interpolation between order
//                       statistics, fp64) of its reliable samples, sorted in
//                       shared memory by a bitonic network.
//   multiwarp_scatter   one CTA per (source frame, target frame): every
//                       source sample is forward-warped, the samples are
//                       counted per target token, warped again and gathered by
//                       token (a counting sort in shared memory), and each
//                       token with at least k_warp samples gets their median
//                       in the workspace (-1 otherwise).
//   multiwarp_select    one thread per target token: the median of the
//                       newest source that has one, else 0 (a hole).
//
// The warp of a sample uses explicitly rounded fp32 operations in the same
// order as the coverage test, so the target token, an integer decided by
// floats, does not depend on FMA contraction.
#include "common.cuh"

namespace velox {
namespace {

__device__ __forceinline__ float mul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float add(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ float sub(float a, float b) { return __fsub_rn(a, b); }
__device__ __forceinline__ float dv(float a, float b) { return __fdiv_rn(a, b); }

constexpr int kThreads = 256;

// ---------------------------------------------------------------- slab table

struct SlabArgs {
  const float *depth;
  const float *conf;     // nullable
  const uint8_t *mask;   // nullable
  int F, frame_base, H, W, s;
  const int32_t *cell_of_rank;
  int n_cells;
  int b, first_block;
  float c_min;
  int n_min;
  double p_lo, p_hi;
  velox_slab *slabs;
  float *token_uvz;      // nullable, s == 1: [n_blocks][b][3]
  int n_pad;             // power of two >= b * s * s
  int32_t *dev_status;
};

__device__ double percentile_sorted(const float *v, int n, double q) {
  const double h = __dmul_rn((double)(n - 1), q);
  const double fl = floor(h);
  const int lo = (int)fl;
  const double t = __dsub_rn(h, fl);
  if (lo + 1 < n) {
    const double a = (double)v[lo], b = (double)v[lo + 1];
    return __dadd_rn(a, __dmul_rn(__dsub_rn(b, a), t));
  }
  return (double)v[lo];
}

__global__ void __launch_bounds__(kThreads) slab_table_kernel(SlabArgs a) {
  extern __shared__ float s_val[];  // [n_pad]
  __shared__ int s_n, s_min[2], s_max[2], s_frame, s_bad;
  const int j = blockIdx.x;
  const int r = a.first_block + j;
  const int HW = a.H * a.W, s = a.s, Ws = a.W * s, Hs = a.H * s;
  if (threadIdx.x == 0) {
    s_n = 0;
    s_min[0] = s_min[1] = INT_MAX;
    s_max[0] = s_max[1] = -1;
    s_bad = 0;
    s_frame = a.cell_of_rank[(size_t)r * a.b] / HW;
  }
  for (int k = threadIdx.x; k < a.n_pad; k += kThreads) s_val[k] = __int_as_float(0x7f800000);
  __syncthreads();
  const int f = s_frame, lf = f - a.frame_base;
  const bool frame_ok = lf >= 0 && lf < a.F;
  const int per_cell = s * s;
  for (int it = threadIdx.x; it < a.b * per_cell; it += kThreads) {
    const int t = it / per_cell, q = it - t * per_cell;
    const int c = a.cell_of_rank[(size_t)r * a.b + t];
    if (c < 0 || c >= a.n_cells || c / HW != f || !frame_ok) {
      s_bad = 1;
      if (a.token_uvz) {
        float *o = a.token_uvz + ((size_t)j * a.b + t) * 3;
        o[0] = o[1] = o[2] = 0.f;
      }
      continue;
    }
    const int rem = c - f * HW, y = rem / a.W, x = rem - y * a.W;
    if (q == 0) {
      atomicMin(&s_min[0], x);
      atomicMin(&s_min[1], y);
      atomicMax(&s_max[0], x);
      atomicMax(&s_max[1], y);
    }
    const int py = y * s + q / s, px = x * s + q % s;
    const size_t idx = ((size_t)lf * Hs + py) * Ws + px;
    const float z = a.depth[idx];
    bool ok = z > 0.f && isfinite(z);
    if (a.mask) ok = ok && a.mask[idx] != 0;
    if (a.conf) ok = ok && a.conf[idx] >= a.c_min;
    if (ok) s_val[atomicAdd(&s_n, 1)] = z;
    if (a.token_uvz) {  // s == 1: token t of the block, its centre and depth
      float *o = a.token_uvz + ((size_t)j * a.b + t) * 3;
      o[0] = (float)x + 0.5f;
      o[1] = (float)y + 0.5f;
      o[2] = ok ? z : 0.f;
    }
  }
  __syncthreads();
  // bitonic sort of s_val[0 .. n_pad) ascending (+inf padding sorts last)
  for (int k = 2; k <= a.n_pad; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < a.n_pad; i += kThreads) {
        const int p = i ^ jj;
        if (p > i) {
          const float x = s_val[i], y = s_val[p];
          const bool up = (i & k) == 0;
          if ((x > y) == up) {
            s_val[i] = y;
            s_val[p] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  if (threadIdx.x == 0) {
    velox_slab out;
    out.cam = f;
    const int n = s_n;
    if (s_bad) flag_error(a.dev_status, VELOX_DEV_BAD_CELL);
    if (!s_bad && n >= a.n_min && n > 0) {
      out.u0 = (float)s_min[0];
      out.u1 = (float)(s_max[0] + 1);
      out.v0 = (float)s_min[1];
      out.v1 = (float)(s_max[1] + 1);
      out.zlo = __double2float_rn(percentile_sorted(s_val, n, a.p_lo));
      out.zhi = __double2float_rn(percentile_sorted(s_val, n, a.p_hi));
      out.valid = 1;
    } else {
      out.u0 = out.u1 = out.v0 = out.v1 = out.zlo = out.zhi = 0.f;
      out.valid = 0;
    }
    a.slabs[j] = out;
  }
}

// ---------------------------------------------------------------- multiwarp

struct WarpArgs {
  const velox_camera *cams;
  int n_cams;
  const float *src_depth;  // [S][H s][W s]
  const int32_t *src_cam;  // [S], newest first
  int S;
  const int32_t *tgt_cam;  // [n_tgt]
  int n_tgt;
  int H, W, s, k_warp;
  float *med;              // workspace [n_tgt][S][H W]: median or -1
  float *zq;               // [n_tgt][H][W]
  int32_t *dev_status;
};

// Target token of source sample (px, py) at depth z, or -1; *dt = target depth.
__device__ __forceinline__ int warp_one(const velox_camera &cs, const velox_camera &ct, int px,
                                        int py, float z, int s, int H, int W, float *dt) {
  const float u = dv(add((float)px, 0.5f), (float)s);
  const float v = dv(add((float)py, 0.5f), (float)s);
  const float x[3] = {mul(dv(sub(u, cs.cx), cs.fx), z), mul(dv(sub(v, cs.cy), cs.fy), z), z};
  float X[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    float acc = mul(cs.R[3 * k + 0], x[0]);
    acc = add(acc, mul(cs.R[3 * k + 1], x[1]));
    acc = add(acc, mul(cs.R[3 * k + 2], x[2]));
    X[k] = add(acc, cs.C[k]);
  }
  const float dx[3] = {sub(X[0], ct.C[0]), sub(X[1], ct.C[1]), sub(X[2], ct.C[2])};
  float d[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    float acc = mul(ct.R[0 + k], dx[0]);
    acc = add(acc, mul(ct.R[3 + k], dx[1]));
    acc = add(acc, mul(ct.R[6 + k], dx[2]));
    d[k] = acc;
  }
  if (!(d[2] > 0.f)) return -1;
  const float pu = add(mul(dv(d[0], d[2]), ct.fx), ct.cx);
  const float pv = add(mul(dv(d[1], d[2]), ct.fy), ct.cy);
  if (!(pu >= 0.f && pu < (float)W && pv >= 0.f && pv < (float)H)) return -1;
  *dt = d[2];
  return (int)floorf(pv) * W + (int)floorf(pu);
}

// Dynamic shared memory: cnt[HW] int, off[HW] int, vals[H s W s] float.
__global__ void __launch_bounds__(kThreads) multiwarp_scatter_kernel(WarpArgs a) {
  extern __shared__ int s_mw[];
  __shared__ int s_part[kThreads];
  const int k = blockIdx.x, tgt = blockIdx.y;
  const int HW = a.H * a.W, Ws = a.W * a.s, n_smp = a.H * a.s * Ws;
  int *cnt = s_mw, *off = s_mw + HW;
  float *vals = reinterpret_cast<float *>(s_mw + 2 * HW);
  float *med = a.med + ((size_t)tgt * a.S + k) * HW;
  const int sc = a.src_cam[k], tc = a.tgt_cam[tgt];
  if (sc < 0 || sc >= a.n_cams || tc < 0 || tc >= a.n_cams) {
    if (threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_BAD_CAMERA);
    for (int t = threadIdx.x; t < HW; t += kThreads) med[t] = -1.f;
    return;
  }
  const velox_camera cs = a.cams[sc], ct = a.cams[tc];
  const float *src = a.src_depth + (size_t)k * n_smp;
  for (int t = threadIdx.x; t < HW; t += kThreads) cnt[t] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n_smp; i += kThreads) {
    const float z = src[i];
    if (!(z > 0.f)) continue;
    float dt;
    const int t = warp_one(cs, ct, i % Ws, i / Ws, z, a.s, a.H, a.W, &dt);
    if (t >= 0) atomicAdd(&cnt[t], 1);
  }
  __syncthreads();
  // exclusive scan of cnt: thread p owns a contiguous run of tokens
  const int run = (HW + kThreads - 1) / kThreads;
  const int lo = min(HW, (int)threadIdx.x * run), hi = min(HW, lo + run);
  int mine = 0;
  for (int t = lo; t < hi; ++t) mine += cnt[t];
  s_part[threadIdx.x] = mine;
  __syncthreads();
  for (int o = 1; o < kThreads; o <<= 1) {
    const int v = threadIdx.x >= (unsigned)o ? s_part[threadIdx.x - o] : 0;
    __syncthreads();
    s_part[threadIdx.x] += v;
    __syncthreads();
  }
  int acc = s_part[threadIdx.x] - mine;
  for (int t = lo; t < hi; ++t) {
    off[t] = acc;
    acc += cnt[t];
  }
  __syncthreads();
  for (int t = threadIdx.x; t < HW; t += kThreads) cnt[t] = 0;  // reused as fill counters
  __syncthreads();
  for (int i = threadIdx.x; i < n_smp; i += kThreads) {
    const float z = src[i];
    if (!(z > 0.f)) continue;
    float dt;
    const int t = warp_one(cs, ct, i % Ws, i / Ws, z, a.s, a.H, a.W, &dt);
    if (t >= 0) vals[off[t] + atomicAdd(&cnt[t], 1)] = dt;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < HW; t += kThreads) {
    const int n = cnt[t];
    float m = -1.f;
    if (n >= a.k_warp) {
      float *v = vals + off[t];
      for (int x = 1; x < n; ++x) {  // insertion sort of this token's samples
        const float key = v[x];
        int y = x - 1;
        while (y >= 0 && v[y] > key) {
          v[y + 1] = v[y];
          --y;
        }
        v[y + 1] = key;
      }
      m = (n & 1) ? v[n / 2]
                  : __double2float_rn(
                        __dmul_rn(__dadd_rn((double)v[n / 2 - 1], (double)v[n / 2]), 0.5));
    }
    med[t] = m;
  }
}

__global__ void multiwarp_select_kernel(WarpArgs a) {
  const int HW = a.H * a.W;
  const int tgt = blockIdx.y;
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= HW) return;
  float z = 0.f;
  for (int k = 0; k < a.S; ++k) {  // newest source first
    const float m = a.med[((size_t)tgt * a.S + k) * HW + t];
    if (m >= 0.f) {
      z = m;
      break;
    }
  }
  a.zq[(size_t)tgt * HW + t] = z;
}

}  // namespace

cudaError_t launch_slab_table(const float *depth, const float *conf, const uint8_t *mask, int F,
                              int frame_base, int H, int W, int s, const int32_t *cell_of_rank,
                              int n_cells, int b, int first_block, int n_blocks, float c_min, int n_min,
                              double p_lo, double p_hi, velox_slab *slabs, float *token_uvz,
                              int32_t *dev_status, cudaStream_t stream) {
  SlabArgs a;
  a.depth = depth;
  a.conf = conf;
  a.mask = mask;
  a.F = F;
  a.frame_base = frame_base;
  a.H = H;
  a.W = W;
  a.s = s;
  a.cell_of_rank = cell_of_rank;
  a.n_cells = n_cells;
  a.b = b;
  a.first_block = first_block;
  a.c_min = c_min;
  a.n_min = n_min;
  a.p_lo = p_lo;
  a.p_hi = p_hi;
  a.slabs = slabs;
  a.token_uvz = token_uvz;
  a.dev_status = dev_status;
  int n_pad = 1;
  while (n_pad < b * s * s) n_pad <<= 1;
  a.n_pad = n_pad;
  const size_t smem = sizeof(float) * (size_t)n_pad;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(slab_table_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  slab_table_kernel<<<n_blocks, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

size_t multiwarp_ws_bytes(int S, int n_tgt, int H, int W) {
  return sizeof(float) * (size_t)S * n_tgt * H * W;
}

cudaError_t launch_multiwarp(const velox_camera *cams, int n_cams, const float *src_depth,
                             const int32_t *src_cam, int S, const int32_t *tgt_cam, int n_tgt,
                             int H, int W, int s, int k_warp, float *zq, void *ws,
                             int32_t *dev_status, cudaStream_t stream) {
  WarpArgs a;
  a.cams = cams;
  a.n_cams = n_cams;
  a.src_depth = src_depth;
  a.src_cam = src_cam;
  a.S = S;
  a.tgt_cam = tgt_cam;
  a.n_tgt = n_tgt;
  a.H = H;
  a.W = W;
  a.s = s;
  a.k_warp = k_warp;
  a.med = static_cast<float *>(ws);
  a.zq = zq;
  a.dev_status = dev_status;
  const size_t smem = sizeof(int) * 2 * (size_t)H * W + sizeof(float) * (size_t)H * W * s * s;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(multiwarp_scatter_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  multiwarp_scatter_kernel<<<dim3(S, n_tgt), kThreads, smem, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  multiwarp_select_kernel<<<dim3((H * W + 255) / 256, n_tgt), 256, 0, stream>>>(a);
  return cudaGetLastError();
}

int multiwarp_max_samples() { return 32768; }
int multiwarp_max_tokens() { return 8192; }
int slab_table_max_samples() { return 16384; }

}  // namespace velox
