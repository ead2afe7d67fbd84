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
//   slab_overlap_kernel   one thread per (query block, history block) pair:
//                         IoU of the two boxes with the intersection counted
//                         on the G^3 cell centres of the query box.  Pairs
//                         whose bounding spheres are apart (with a margin
//                         far above rounding) are 0 without sampling.
//   coverage_kernel       one CTA per query block: every token's warped depth
//                         is back-projected and tested against the past slabs
//                         (rectangle and depth range in the slab's camera);
//                         rho = covered tokens / b, covered = rho >= eta.
//
// Every inside/outside decision uses explicitly rounded fp32 operations
// (__fmul_rn, __fadd_rn, __fsub_rn, __fdiv_rn) in a fixed order, so no
// contraction into FMA changes which side of a face a point lands on.
#include "common.cuh"

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

__global__ void __launch_bounds__(256) slab_overlap_kernel(const velox_camera *__restrict__ cams,
                                                           int n_cams,
                                                           const velox_slab *__restrict__ qs,
                                                           int N,
                                                           const velox_slab *__restrict__ hs,
                                                           int M, int G, float *__restrict__ g,
                                                           int32_t *dev_status) {
  const int i = blockIdx.y;
  const int r = blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= M) return;
  const velox_slab sq = qs[i], sr = hs[r];
  float out = 0.f;
  if (sr.valid && sq.cam >= 0 && sq.cam < n_cams && sr.cam >= 0 && sr.cam < n_cams) {
    const Box bi = make_box(cams[sq.cam], sq);
    const Box br = make_box(cams[sr.cam], sr);
    const float dx = bi.c[0] - br.c[0], dy = bi.c[1] - br.c[1], dz = bi.c[2] - br.c[2];
    const float ri = sqrtf(bi.h[0] * bi.h[0] + bi.h[1] * bi.h[1] + bi.h[2] * bi.h[2]);
    const float rr = sqrtf(br.h[0] * br.h[0] + br.h[1] * br.h[1] + br.h[2] * br.h[2]);
    const float reach = (ri + rr) * 1.001f + 1e-6f;
    if (dx * dx + dy * dy + dz * dz <= reach * reach) {
      int n_in = 0;
      for (int a = 0; a < G; ++a) {
        const float sa = sub(dv((float)(2 * a + 1), (float)G), 1.0f);
        for (int b = 0; b < G; ++b) {
          const float sb = sub(dv((float)(2 * b + 1), (float)G), 1.0f);
          for (int c = 0; c < G; ++c) {
            const float sc = sub(dv((float)(2 * c + 1), (float)G), 1.0f);
            const float p[3] = {mul(sa, bi.h[0]), mul(sb, bi.h[1]), mul(sc, bi.h[2])};
            float X[3], d[3];
            cam_to_world(bi.R, bi.c, p, X);
            world_to_local(br.R, br.c, X, d);
            n_in += (fabsf(d[0]) <= br.h[0] && fabsf(d[1]) <= br.h[1] && fabsf(d[2]) <= br.h[2]);
          }
        }
      }
      const float vi = 8.0f * bi.h[0] * bi.h[1] * bi.h[2];
      const float vr = 8.0f * br.h[0] * br.h[1] * br.h[2];
      const float inter = vi * ((float)n_in / (float)(G * G * G));
      const float uni = vi + vr - inter;
      out = uni > 0.f ? inter / uni : 0.f;
    }
  } else if (sr.valid) {
    flag_error(dev_status, VELOX_DEV_BAD_CAMERA);
  }
  g[(size_t)i * M + r] = out;
}

// One CTA per query block, blockDim = b * kParts: thread (t, part) tests
// token t against the slabs r = part, part + kParts, ...
constexpr int kParts = 8;

__global__ void coverage_kernel(const velox_camera *__restrict__ cams, int n_cams,
                                const velox_slab *__restrict__ qs, const float *__restrict__ q_uvz,
                                int b, const velox_slab *__restrict__ hs, int M, float eta,
                                float *__restrict__ rho, uint8_t *__restrict__ covered,
                                int32_t *dev_status) {
  extern __shared__ int s_cov_raw[];
  volatile int *s_cov = s_cov_raw;  // [b] per-token covered flags (read by other parts)
  const int i = blockIdx.x;
  const int t = threadIdx.x % b, part = threadIdx.x / b;
  for (int k = threadIdx.x; k < b; k += blockDim.x) s_cov[k] = 0;
  __syncthreads();
  const velox_slab sq = qs[i];
  if (sq.cam >= 0 && sq.cam < n_cams) {
    const velox_camera ct = cams[sq.cam];
    const float u = q_uvz[((size_t)i * b + t) * 3 + 0];
    const float v = q_uvz[((size_t)i * b + t) * 3 + 1];
    const float z = q_uvz[((size_t)i * b + t) * 3 + 2];
    if (z > 0.f) {
      const float x[3] = {mul(dv(sub(u, ct.cx), ct.fx), z), mul(dv(sub(v, ct.cy), ct.fy), z), z};
      float X[3];
      cam_to_world(ct.R, ct.C, x, X);
      for (int r = part; r < M; r += kParts) {
        if (s_cov[t]) break;  // another part already covered this token
        const velox_slab sr = hs[r];
        if (!sr.valid) continue;
        if (sr.cam < 0 || sr.cam >= n_cams) {
          flag_error(dev_status, VELOX_DEV_BAD_CAMERA);
          continue;
        }
        const velox_camera &cr = cams[sr.cam];
        float d[3];
        world_to_local(cr.R, cr.C, X, d);  // camera frame of the slab's camera
        if (!(d[2] > 0.f)) continue;
        const float pu = add(mul(dv(d[0], d[2]), cr.fx), cr.cx);
        const float pv = add(mul(dv(d[1], d[2]), cr.fy), cr.cy);
        if (sr.u0 <= pu && pu < sr.u1 && sr.v0 <= pv && pv < sr.v1 && sr.zlo <= d[2] &&
            d[2] <= sr.zhi) {
          s_cov[t] = 1;
          break;
        }
      }
    }
  } else if (threadIdx.x == 0) {
    flag_error(dev_status, VELOX_DEV_BAD_CAMERA);
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    int n = 0;
    for (int k = threadIdx.x; k < b; k += 32) n += s_cov[k];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
    if (threadIdx.x == 0) {
      const float rh = (float)n / (float)b;
      rho[i] = rh;
      covered[i] = rh >= eta ? 1 : 0;
    }
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
  coverage_kernel<<<N, b * kParts, b * sizeof(int), stream>>>(cams, n_cams, qs, q_uvz, b, hs, M,
                                                              eta, rho, covered, dev_status);
  return cudaGetLastError();
}

}  // namespace velox
