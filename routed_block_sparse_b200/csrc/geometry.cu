// Frustum-slab overlap g_{i,r} and coverage rho_i: the geometric inputs of
// the route build.
//
// Velox project page, "02 · Method", steps 01-02 and the glossary entry for
// g; digest of arXiv 2610.22311, "Prerequisites" (frustum slab, OBB overlap)
// and "Method steps", steps one to three (Eq. 7-8); onedev.kr summary, "How
// it differs".  A slab is a token rectangle of a source camera plus a depth
// interval; it is approximated by a camera-facing oriented box whose centre
// lies on the ray through the rectangle centre at the mid depth.
//
//   slab_overlap_kernel   one thread per (query block, history block) pair
//                         decides whether the pair can overlap (bounding
//                         spheres, with a margin far above rounding); the
//                         warp then counts the G^3 cell centres of the query
//                         box inside the history box for each candidate of
//                         its 32 together.
//   coverage_kernel       a cluster of 4 CTAs per query block, each taking a
//                         quarter of its tokens: every token's warped depth
//                         is back-projected and tested against the past slabs
//                         (rectangle and depth range in the slab's camera);
//                         rho = covered tokens / b, covered = rho >= eta.
//                         Slabs whose frustum's bounding sphere cannot reach
//                         the block's token cloud are dropped first (with a
//                         margin far above rounding, so no decision changes);
//                         a token's projection into a camera is formed once
//                         for a run of slabs of that camera; the quarters'
//                         covered counts meet in CTA 0's shared memory.
//
// Every inside/outside decision uses explicitly rounded fp32 operations
// (__fmul_rn, __fadd_rn, __fsub_rn, __fdiv_rn) in a fixed order, so no
// contraction into FMA changes which side of a face a point lands on.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace velox {
namespace {

struct Box {
  float c[3];   // centre
  float R[9];   // axes (columns), row-major storage of the camera rotation
  float h[3];   // half extents
};

__device__ __forceinline__ float mul(float a, float b) { return __fmul_rn(a, b); }
__device__ __forceinline__ float add(float a, float b) { return __fadd_rn(a, b); }
__device__ __forceinline__ float sub(float a, float b) { return __fsub_rn(a, b); }
__device__ __forceinline__ float dv(float a, float b) { return __fdiv_rn(a, b); }

// C + R x, rounded as ((R0 x0 + R1 x1) + R2 x2) + C per component
__device__ __forceinline__ void cam_to_world(const float *R, const float *C, const float *x,
                                             float *X) {
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    float acc = mul(R[3 * k + 0], x[0]);
    acc = add(acc, mul(R[3 * k + 1], x[1]));
    acc = add(acc, mul(R[3 * k + 2], x[2]));
    X[k] = add(acc, C[k]);
  }
}
// R^T (X - c), same rounding order
__device__ __forceinline__ void world_to_local(const float *R, const float *c, const float *X,
                                               float *d) {
  const float dx[3] = {sub(X[0], c[0]), sub(X[1], c[1]), sub(X[2], c[2])};
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    float acc = mul(R[0 + k], dx[0]);
    acc = add(acc, mul(R[3 + k], dx[1]));
    acc = add(acc, mul(R[6 + k], dx[2]));
    d[k] = acc;
  }
}

__device__ Box make_box(const velox_camera &cam, const velox_slab &s) {
  Box b;
  const float zm = mul(0.5f, add(s.zlo, s.zhi));
  const float um = mul(0.5f, add(s.u0, s.u1));
  const float vm = mul(0.5f, add(s.v0, s.v1));
  const float x[3] = {mul(dv(sub(um, cam.cx), cam.fx), zm), mul(dv(sub(vm, cam.cy), cam.fy), zm),
                      zm};
#pragma unroll
  for (int k = 0; k < 9; ++k) b.R[k] = cam.R[k];
  cam_to_world(cam.R, cam.C, x, b.c);
  b.h[0] = mul(dv(mul(sub(s.u1, s.u0), 0.5f), cam.fx), zm);
  b.h[1] = mul(dv(mul(sub(s.v1, s.v0), 0.5f), cam.fy), zm);
  b.h[2] = mul(0.5f, sub(s.zhi, s.zlo));
  return b;
}

// Conservative separating-axis test: true only when the two boxes are apart
// along one of the 15 axes (3 + 3 face normals, 9 edge cross products) by a
// gap far above the rounding of the sampled inside tests, so a pair it
// rejects would have counted no sample inside.  Cross products of nearly
// parallel edges are short and can only fail to separate.
__device__ bool boxes_apart(const Box &a, const Box &b) {
  const float T[3] = {b.c[0] - a.c[0], b.c[1] - a.c[1], b.c[2] - a.c[2]};
  float A[3][3], B[3][3];  // A[k] = axis k of box a (column k of its rotation)
#pragma unroll
  for (int k = 0; k < 3; ++k)
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      A[k][j] = a.R[3 * j + k];
      B[k][j] = b.R[3 * j + k];
    }
  const float tn = sqrtf(T[0] * T[0] + T[1] * T[1] + T[2] * T[2]);
  // world-coordinate scale of the sampled points: their rounding is relative to it
  const float sc = 1.f + fmaxf(fmaxf(fabsf(a.c[0]), fabsf(a.c[1])), fabsf(a.c[2])) +
                   fmaxf(fmaxf(fabsf(b.c[0]), fabsf(b.c[1])), fabsf(b.c[2])) +
                   a.h[0] + a.h[1] + a.h[2] + b.h[0] + b.h[1] + b.h[2];
  auto apart = [&](const float *L) {
    float t = fabsf(L[0] * T[0] + L[1] * T[1] + L[2] * T[2]);
    float r = 0.f;
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      r += a.h[k] * fabsf(L[0] * A[k][0] + L[1] * A[k][1] + L[2] * A[k][2]);
      r += b.h[k] * fabsf(L[0] * B[k][0] + L[1] * B[k][1] + L[2] * B[k][2]);
    }
    const float ln = sqrtf(L[0] * L[0] + L[1] * L[1] + L[2] * L[2]);
    return t - r > 1e-4f * (r + tn * ln) + 1e-5f * sc * ln;
  };
#pragma unroll
  for (int k = 0; k < 3; ++k) {
    if (apart(A[k]) || apart(B[k])) return true;
  }
#pragma unroll
  for (int k = 0; k < 3; ++k)
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      const float L[3] = {A[k][1] * B[j][2] - A[k][2] * B[j][1], A[k][2] * B[j][0] - A[k][0] * B[j][2],
                          A[k][0] * B[j][1] - A[k][1] * B[j][0]};
      if (apart(L)) return true;
    }
  return false;
}

// Sample points of the query box inside the history box, lane's share: lane
// takes the (b, c) index pairs lane, lane + 32, ... and walks a.  off[k] =
// (2k + 1) / G - 1.  The products R x of cam_to_world that do not depend on
// a are formed once per pair; every value is the one the plain per-point
// evaluation rounds to.
__device__ __forceinline__ int count_inside(const Box &bi, const Box &br, int G,
                                            const float *off, int lane) {
  int n_in = 0;
  for (int bc = lane; bc < G * G; bc += 32) {
    const int bb = bc / G, cc = bc - bb * G;
    const float p1 = mul(off[bb], bi.h[1]), p2 = mul(off[cc], bi.h[2]);
    float q1[3], q2[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      q1[k] = mul(bi.R[3 * k + 1], p1);
      q2[k] = mul(bi.R[3 * k + 2], p2);
    }
    for (int a = 0; a < G; ++a) {
      const float p0 = mul(off[a], bi.h[0]);
      float dx[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        float acc = add(mul(bi.R[3 * k + 0], p0), q1[k]);
        acc = add(acc, q2[k]);
        dx[k] = sub(add(acc, bi.c[k]), br.c[k]);
      }
      bool in = true;
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        float acc = mul(br.R[0 + k], dx[0]);
        acc = add(acc, mul(br.R[3 + k], dx[1]));
        acc = add(acc, mul(br.R[6 + k], dx[2]));
        in = in && fabsf(acc) <= br.h[k];
      }
      n_in += in;
    }
  }
  return n_in;
}

// Thread per (query block i, history block r) decides whether the pair can
// overlap (valid slab, cameras in range, boxes not apart); then the warp
// samples each candidate pair of its 32 together and the candidate's own
// lane writes the ratio.
__global__ void __launch_bounds__(256) slab_overlap_kernel(const velox_camera *__restrict__ cams,
                                                           int n_cams,
                                                           const velox_slab *__restrict__ qs,
                                                           int N,
                                                           const velox_slab *__restrict__ hs,
                                                           int M, int G, float *__restrict__ g,
                                                           int32_t *dev_status) {
  __shared__ float s_off[32];
  const int i = blockIdx.y;
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < G) s_off[threadIdx.x] = sub(dv((float)(2 * threadIdx.x + 1), (float)G), 1.0f);
  __syncthreads();
  const velox_slab sq = qs[i];
  const bool q_ok = sq.cam >= 0 && sq.cam < n_cams;
  Box bi;
  if (q_ok) bi = make_box(cams[sq.cam], sq);
  bool cand = false;
  if (r < M) {
    const velox_slab sr = hs[r];
    if (sr.valid && q_ok && sr.cam >= 0 && sr.cam < n_cams) {
      cand = !boxes_apart(bi, make_box(cams[sr.cam], sr));
    } else if (sr.valid) {
      flag_error(dev_status, VELOX_DEV_BAD_CAMERA);
    }
  }
  float out = 0.f;
  unsigned pending = __ballot_sync(0xffffffffu, cand);
  while (pending) {
    const int src = __ffs(pending) - 1;
    pending &= pending - 1;
    const velox_slab sr = hs[(r - lane) + src];
    const Box br = make_box(cams[sr.cam], sr);
    int n_in = count_inside(bi, br, G, s_off, lane);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n_in += __shfl_xor_sync(0xffffffffu, n_in, off);
    if (lane == src) {
      const float vi = 8.0f * bi.h[0] * bi.h[1] * bi.h[2];
      const float vr = 8.0f * br.h[0] * br.h[1] * br.h[2];
      const float inter = vi * ((float)n_in / (float)(G * G * G));
      const float uni = vi + vr - inter;
      out = uni > 0.f ? inter / uni : 0.f;
    }
  }
  if (r < M) g[(size_t)i * M + r] = out;
}

// A cluster of kSplit CTAs per query block; CTA q takes tokens
// [q tpc, (q + 1) tpc) with tpc = ceil(b / kSplit), and tpc * kParts working
// threads (rounded up to whole warps): thread (t, part) tests token t against
// the part-th contiguous share of the surviving slabs.
constexpr int kSplit = 4;
constexpr int kParts = 32;
constexpr int kSlabChunk = 2048;  // slabs culled and tested per round

// World corner k (bit 0: u, bit 1: v, bit 2: depth) of a slab's frustum.
__device__ __forceinline__ void frustum_corner(const velox_camera &c, const velox_slab &s, int k,
                                               float *X) {
  const float u = (k & 1) ? s.u1 : s.u0, v = (k & 2) ? s.v1 : s.v0;
  const float z = (k & 4) ? s.zhi : s.zlo;
  const float x[3] = {(u - c.cx) / c.fx * z, (v - c.cy) / c.fy * z, z};
  cam_to_world(c.R, c.C, x, X);
}

__global__ void __cluster_dims__(kSplit, 1, 1) __launch_bounds__(1024)
    coverage_kernel(const velox_camera *__restrict__ cams, int n_cams,
                                const velox_slab *__restrict__ qs, const float *__restrict__ q_uvz,
                                int b, const velox_slab *__restrict__ hs, int M, float eta,
                                float *__restrict__ rho, uint8_t *__restrict__ covered,
                                int32_t *dev_status) {
  extern __shared__ int s_cov_raw[];
  volatile int *s_cov = s_cov_raw;  // [tpc] per-token covered flags (read by other parts)
  __shared__ int s_list[kSlabChunk];
  __shared__ int s_nlist;
  __shared__ float s_red[32][4];
  __shared__ float s_sphere[4];  // token cloud centre and radius
  __shared__ int s_total;        // CTA 0 of the cluster: covered tokens of the block
  cg::cluster_group cluster = cg::this_cluster();
  const int q = (int)cluster.block_rank();
  const int i = blockIdx.x / kSplit;
  const int tpc = (b + kSplit - 1) / kSplit;
  const int tl = threadIdx.x % tpc, part = threadIdx.x / tpc;
  const int t = q * tpc + tl;  // token of the block
  const bool act = part < kParts && t < b;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int k = threadIdx.x; k < tpc; k += blockDim.x) s_cov[k] = 0;
  if (threadIdx.x == 0) s_total = 0;
  const velox_slab sq = qs[i];
  const bool q_ok = sq.cam >= 0 && sq.cam < n_cams;
  if (!q_ok && threadIdx.x == 0 && q == 0) flag_error(dev_status, VELOX_DEV_BAD_CAMERA);
  float X[3] = {0.f, 0.f, 0.f};
  bool live = false;
  if (q_ok && act) {
    const velox_camera &ct = cams[sq.cam];
    const float u = q_uvz[((size_t)i * b + t) * 3 + 0];
    const float v = q_uvz[((size_t)i * b + t) * 3 + 1];
    const float z = q_uvz[((size_t)i * b + t) * 3 + 2];
    if (z > 0.f) {
      const float x[3] = {mul(dv(sub(u, ct.cx), ct.fx), z), mul(dv(sub(v, ct.cy), ct.fy), z), z};
      cam_to_world(ct.R, ct.C, x, X);
      live = true;
    }
  }
  // bounding sphere of the block's live token points (parts 0 only count)
  {
    const bool own = live && part == 0;
    float a0 = own ? X[0] : 0.f, a1 = own ? X[1] : 0.f, a2 = own ? X[2] : 0.f;
    float n = own ? 1.f : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      a0 += __shfl_xor_sync(0xffffffffu, a0, off);
      a1 += __shfl_xor_sync(0xffffffffu, a1, off);
      a2 += __shfl_xor_sync(0xffffffffu, a2, off);
      n += __shfl_xor_sync(0xffffffffu, n, off);
    }
    if (lane == 0) { s_red[warp][0] = a0; s_red[warp][1] = a1; s_red[warp][2] = a2; s_red[warp][3] = n; }
    __syncthreads();
    if (threadIdx.x == 0) {
      float c0 = 0.f, c1 = 0.f, c2 = 0.f, cn = 0.f;
      for (int w = 0; w < nwarps; ++w) { c0 += s_red[w][0]; c1 += s_red[w][1]; c2 += s_red[w][2]; cn += s_red[w][3]; }
      cn = cn > 0.f ? cn : 1.f;
      s_sphere[0] = c0 / cn; s_sphere[1] = c1 / cn; s_sphere[2] = c2 / cn;
    }
    __syncthreads();
    float d2 = 0.f;
    if (own) {
      const float e0 = X[0] - s_sphere[0], e1 = X[1] - s_sphere[1], e2 = X[2] - s_sphere[2];
      d2 = e0 * e0 + e1 * e1 + e2 * e2;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) d2 = fmaxf(d2, __shfl_xor_sync(0xffffffffu, d2, off));
    __syncthreads();
    if (lane == 0) s_red[warp][0] = d2;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = 0.f;
      for (int w = 0; w < nwarps; ++w) m = fmaxf(m, s_red[w][0]);
      s_sphere[3] = sqrtf(m);
    }
    __syncthreads();
  }
  const float tc0 = s_sphere[0], tc1 = s_sphere[1], tc2 = s_sphere[2], trad = s_sphere[3];
  __shared__ int s_wcnt[32];
  for (int base = 0; base < M; base += kSlabChunk) {
    const int hi = min(M, base + kSlabChunk);
    if (threadIdx.x == 0) s_nlist = 0;
    __syncthreads();
    // keep the slabs whose frustum's bounding sphere reaches the token cloud
    // (a token inside a frustum lies inside its sphere, and the margin
    // covers every rounding of the inside test), compacted in id order so
    // that slabs of one camera stay together
    for (int sub0 = base; sub0 < hi; sub0 += blockDim.x) {
      const int r = sub0 + threadIdx.x;
      bool keep = false;
      if (r < hi && q_ok) {
        const velox_slab sr = hs[r];
        if (sr.valid && (sr.cam < 0 || sr.cam >= n_cams)) {
          flag_error(dev_status, VELOX_DEV_BAD_CAMERA);
        } else if (sr.valid) {
          const velox_camera &cr = cams[sr.cam];
          float P[8][3], m0 = 0.f, m1 = 0.f, m2 = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            frustum_corner(cr, sr, k, P[k]);
            m0 += P[k][0]; m1 += P[k][1]; m2 += P[k][2];
          }
          m0 *= 0.125f; m1 *= 0.125f; m2 *= 0.125f;
          float rr = 0.f;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float e0 = P[k][0] - m0, e1 = P[k][1] - m1, e2 = P[k][2] - m2;
            rr = fmaxf(rr, e0 * e0 + e1 * e1 + e2 * e2);
          }
          const float e0 = m0 - tc0, e1 = m1 - tc1, e2 = m2 - tc2;
          const float reach =
              (sqrtf(rr) + trad) * 1.001f + 1e-4f * (1.f + fabsf(m0) + fabsf(m1) + fabsf(m2));
          keep = e0 * e0 + e1 * e1 + e2 * e2 <= reach * reach;
        }
      }
      const unsigned bal = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) s_wcnt[warp] = __popc(bal);
      __syncthreads();
      int before = s_nlist, total = 0;
      for (int w = 0; w < nwarps; ++w) {
        if (w < warp) before += s_wcnt[w];
        total += s_wcnt[w];
      }
      if (keep) s_list[before + __popc(bal & ((1u << lane) - 1u))] = r;
      __syncthreads();
      if (threadIdx.x == 0) s_nlist += total;
      __syncthreads();
    }
    const int nl = s_nlist;
    if (live) {
      // part p takes a contiguous share of the list; the projection into a
      // camera is formed once for a run of slabs of that camera (the values
      // are the ones each slab's own test would compute)
      const int per = (nl + kParts - 1) / kParts;
      const int k1 = min(nl, (part + 1) * per);
      int last_cam = -1;
      bool front = false;
      float pu = 0.f, pv = 0.f, dz = 0.f;
      for (int k = part * per; k < k1; ++k) {
        if (s_cov[tl]) break;  // another part already covered this token
        const velox_slab sr = hs[s_list[k]];
        if (sr.cam != last_cam) {
          last_cam = sr.cam;
          const velox_camera &cr = cams[sr.cam];
          float d[3];
          world_to_local(cr.R, cr.C, X, d);  // camera frame of the slab's camera
          dz = d[2];
          front = d[2] > 0.f;
          if (front) {
            pu = add(mul(dv(d[0], d[2]), cr.fx), cr.cx);
            pv = add(mul(dv(d[1], d[2]), cr.fy), cr.cy);
          }
        }
        if (front && sr.zlo <= dz && dz <= sr.zhi && sr.u0 <= pu && pu < sr.u1 && sr.v0 <= pv &&
            pv < sr.v1) {
          s_cov[tl] = 1;
          break;
        }
      }
    }
    __syncthreads();
  }
  // every CTA's s_total is initialised before any CTA adds to CTA 0's
  cluster.sync();
  if (threadIdx.x < 32) {
    int n = 0;
    for (int k = threadIdx.x; k < tpc; k += 32) n += s_cov[k];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
    if (threadIdx.x == 0) atomicAdd(cluster.map_shared_rank(&s_total, 0), n);
  }
  cluster.sync();
  if (q == 0 && threadIdx.x == 0) {
    const float rh = (float)s_total / (float)b;
    rho[i] = rh;
    covered[i] = rh >= eta ? 1 : 0;
  }
}

}  // namespace

cudaError_t launch_slab_overlap(const velox_camera *cams, int n_cams, const velox_slab *qs, int N,
                                const velox_slab *hs, int M, int G, float *g,
                                int32_t *dev_status, cudaStream_t stream) {
  dim3 grid((M + 255) / 256, N);
  slab_overlap_kernel<<<grid, 256, 0, stream>>>(cams, n_cams, qs, N, hs, M, G, g, dev_status);
  return cudaGetLastError();
}

cudaError_t launch_coverage(const velox_camera *cams, int n_cams, const velox_slab *qs,
                            const float *q_uvz, int N, int b, const velox_slab *hs, int M,
                            float eta, float *rho, uint8_t *covered, int32_t *dev_status,
                            cudaStream_t stream) {
  const int tpc = (b + kSplit - 1) / kSplit;
  const int threads = (tpc * kParts + 31) / 32 * 32;
  coverage_kernel<<<N * kSplit, threads, tpc * sizeof(int), stream>>>(cams, n_cams, qs, q_uvz, b,
                                                                      hs, M, eta, rho, covered,
                                                                      dev_status);
  return cudaGetLastError();
}

}  // namespace velox
