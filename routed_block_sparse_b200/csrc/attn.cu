// Index-based block-sparse attention over routed 128-token KV tiles.
//
// Digest of arXiv 2610.22311, "Core method" (Eq. 15) and "Novelty"; Velox
// project page, "Why the route is a block, not a token": the kernel visits
// only the KV tiles listed in a query block's route, so a skipped tile saves
// both its QK^T product and its K/V load.  The result is an ordinary softmax
// attention restricted to the tokens of the listed tiles, computed with the
// FlashAttention online-softmax recurrence over tiles.
//
// sm_100a design: one CTA per (head, query block), two CTAs per SM.  Within a
// CTA the chain S_j -> softmax_j -> PV_j is serial (P lives in the TMEM
// columns of S), and the second CTA on the SM fills the tensor core while the
// first one runs its softmax, so the two query blocks ping-pong on the SM.
//   warp 0      TMA producer: Q once, then the K and V tiles of the route
//               (128-byte swizzle, two 64-channel boxes per tile); K_{j+1} is
//               fetched as soon as S_j is done, V_{j+1} as soon as PV_j is.
//   warp 1      TMEM allocator (256 columns: S/P 128, O 128) and the single
//               tcgen05.mma issuer: S_j = Q K_j^T (A, B from shared memory),
//               O += P_j V_j (A = P from TMEM, B = V from shared memory).
//   warps 2-5   softmax: one query row per thread (its TMEM lane).  Row max
//               with independent partial maxima, exponentials in the log2
//               domain, P_j packed to bf16 into the S columns with
//               tcgen05.st.  The running max is only moved (and O rescaled in
//               TMEM) when it grows by more than 2^8; otherwise the stale max
//               is kept, which is exact because O and the row sum always use
//               the same max.  Epilogue: O / l -> bf16, lse.
// A pre-pass compacts the route into shared memory, skipping ids outside
// [0, M) and repeats (flagged in dev_status).
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"

namespace velox {
namespace {

constexpr int BM = 128;  // query rows per tile
constexpr int BN = 128;  // tokens per KV tile
constexpr int D = 128;   // head dim
constexpr int kThreads = 192;
constexpr uint32_t kTileBytes = BN * D * 2;      // 32 KB
constexpr uint32_t kHalfBytes = kTileBytes / 2;  // one 64-channel box
constexpr int kMaxRoute = VELOX_MAX_ROUTE;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColS = 0;    // S (fp32, 128 columns); P (bf16x2) in its first 64
constexpr uint32_t kColO = 128;  // O accumulator (fp32, 128 columns)
constexpr float kRescaleThreshold = 8.0f;  // log2 of the largest tolerated growth

// shared-memory layout (offsets from a 1024-byte aligned base)
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;
constexpr uint32_t kOffV = kOffK + kTileBytes;
constexpr uint32_t kOffBar = kOffV + kTileBytes;
constexpr uint32_t kNumBars = 10;
constexpr uint32_t kOffMisc = kOffBar + kNumBars * 8;
constexpr uint32_t kOffDyn = kOffMisc + 64;  // route list (uint16), then the id bitmap

struct AttnArgs {
  const int32_t *route_ids;  // null: dense
  const int32_t *route_len;
  int R_max;
  int N, M;
  float scale_log2;  // softmax_scale * log2(e)
  uint16_t *O;
  float *lse;
  int32_t *dev_status;
  uint32_t bits_offset;  // byte offset of the id bitmap from the aligned base
};

__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile_saddr, int k) {
  // K-major operand, 128-byte swizzle: 16-element K steps advance 32 bytes
  // inside a 64-element atom; atoms (64 channels) are 16 KB apart.
  return smem_desc_sw128(tile_saddr + (k >> 2) * kHalfBytes + (k & 3) * 32, 16, 1024);
}
__device__ __forceinline__ uint64_t vmn_desc(uint32_t tile_saddr, int k) {
  // V as the MN-major B operand (N = channel, K = token): 16-token K steps
  // advance 16 rows of 128 bytes; the two 64-channel halves are 16 KB apart.
  return smem_desc_sw128(tile_saddr + k * 16 * 128, kHalfBytes, 1024);
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16: A (P, bf16) read from TMEM.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-uniform bounded wait (tcgen05.ld/st after it are warp-collective).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort));
}

__global__ void __launch_bounds__(kThreads, 2)
    attn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                const __grid_constant__ CUtensorMap tmV, AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  uint8_t *sQ = base + kOffQ;
  uint8_t *sK = base + kOffK;
  uint8_t *sV = base + kOffV;
  uint64_t *bar = reinterpret_cast<uint64_t *>(base + kOffBar);
  uint64_t *q_full = bar + 0, *k_full = bar + 1, *k_empty = bar + 2, *v_full = bar + 3,
           *v_empty = bar + 4, *s_full = bar + 5, *p_full = bar + 6, *o_done = bar + 7,
           *mma_done = bar + 8;
  uint32_t *s_tmem = reinterpret_cast<uint32_t *>(base + kOffMisc);
  int *s_nvalid = reinterpret_cast<int *>(base + kOffMisc + 4);
  volatile int *s_abort = reinterpret_cast<volatile int *>(base + kOffMisc + 8);
  uint16_t *tiles = reinterpret_cast<uint16_t *>(base + kOffDyn);
  uint32_t *bits = reinterpret_cast<uint32_t *>(base + a.bits_offset);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x;
  const int h = row / a.N, i = row - h * a.N;
  const bool dense = (a.route_ids == nullptr);
  const int M = a.M;

  // ---- set-up: barriers, TMEM, route compaction
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(k_full, 1);
    mbar_init(k_empty, 1);
    mbar_init(v_full, 1);
    mbar_init(v_empty, 1);
    mbar_init(s_full, 1);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(mma_done, 1);
    *s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  int L = 0;
  if (!dense) {
    L = a.route_len[row];
    if (L < 0 || L > a.R_max) {
      if (threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_ROUTE_LEN);
      L = 0;
    }
    const int W = (M + 31) >> 5;
    for (int k = threadIdx.x; k < W; k += kThreads) bits[k] = 0u;
  }
  __syncthreads();
  if (warp == 0) {
    if (dense) {
      if (lane == 0) *s_nvalid = M;
    } else {
      const int32_t *ids = a.route_ids + (size_t)row * a.R_max;
      int n = 0;
      bool bad = false, dup = false;
      for (int b0 = 0; b0 < L; b0 += 32) {
        const int j = b0 + lane;
        const int id = j < L ? ids[j] : -1;
        bool ok = (j < L) && id >= 0 && id < M;
        if (j < L && !ok) bad = true;
        if (ok) {
          const uint32_t m = 1u << (id & 31);
          if (atomicOr(&bits[id >> 5], m) & m) {
            ok = false;
            dup = true;
          }
        }
        const unsigned vote = __ballot_sync(0xffffffffu, ok);
        if (ok) tiles[n + __popc(vote & ((1u << lane) - 1u))] = static_cast<uint16_t>(id);
        n += __popc(vote);
      }
      if (__any_sync(0xffffffffu, bad) && lane == 0) flag_error(a.dev_status, VELOX_DEV_BAD_ROUTE_ID);
      if (__any_sync(0xffffffffu, dup) && lane == 0) flag_error(a.dev_status, VELOX_DEV_DUP_ROUTE_ID);
      if (lane == 0) *s_nvalid = n;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const int n = *s_nvalid;
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    // ================= TMA producer =================
    if (lane == 0 && n > 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_3d(sQ, &tmQ, q_full, 0, i * BM, h);
      tma_load_3d(sQ + kHalfBytes, &tmQ, q_full, 64, i * BM, h);
      int k_issued = 0, v_issued = 0;
      for (int j = 0; j < n; ++j) {
        const uint32_t free_parity = (j & 1) ^ 1;
        const int tile = dense ? j : tiles[j];
        if (!mbar_wait(k_empty, free_parity, s_abort)) break;
        mbar_arrive_expect_tx(k_full, kTileBytes);
        tma_load_3d(sK, &tmK, k_full, 0, tile * BN, h);
        tma_load_3d(sK + kHalfBytes, &tmK, k_full, 64, tile * BN, h);
        k_issued = j + 1;
        if (!mbar_wait(v_empty, free_parity, s_abort)) break;
        mbar_arrive_expect_tx(v_full, kTileBytes);
        tma_load_3d(sV, &tmV, v_full, 0, tile * BN, h);
        tma_load_3d(sV + kHalfBytes, &tmV, v_full, 64, tile * BN, h);
        v_issued = j + 1;
      }
      if (*s_abort) {
        // let the copies already in flight land before the CTA goes away
        // (each wait is bounded by the same time limit)
        volatile int never = 0;
        mbar_wait(q_full, 0, &never);
        if (k_issued > 0) {
          never = 0;
          mbar_wait(k_full, (k_issued - 1) & 1, &never);
        }
        if (v_issued > 0) {
          never = 0;
          mbar_wait(v_full, (v_issued - 1) & 1, &never);
        }
      }
    }
  } else if (warp == 1) {
    // ================= MMA issuer =================
    if (lane == 0 && n > 0) {
      constexpr uint32_t idS = idesc_bf16_f32(BM, BN, false);
      constexpr uint32_t idPV = idesc_bf16_f32(BM, D, true);
      const uint32_t qa = smem_u32(sQ), ka = smem_u32(sK), va = smem_u32(sV);
      bool ok = mbar_wait(q_full, 0, s_abort);
      for (int j = 0; ok && j < n; ++j) {
        const uint32_t ph = j & 1;
        if (!mbar_wait(k_full, ph, s_abort)) break;
        // S_j overwrites the columns P_{j-1} was read from
        if (j > 0 && !mbar_wait(o_done, ph ^ 1, s_abort)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < D / 16; ++k)
          mma_bf16_ss(tmem + kColS, kmajor_desc(qa, k), kmajor_desc(ka, k), idS, k > 0);
        tc_commit(s_full);
        tc_commit(k_empty);
        if (!mbar_wait(p_full, ph, s_abort)) break;
        if (!mbar_wait(v_full, ph, s_abort)) break;
        tc_fence_after();
#pragma unroll
        for (int k = 0; k < BN / 16; ++k)
          mma_bf16_ts(tmem + kColO, tmem + kColS + k * 8, vmn_desc(va, k), idPV,
                      (j > 0 || k > 0));
        tc_commit(o_done);
        tc_commit(v_empty);
      }
      // all issued MMAs must be complete before TMEM is released
      tc_commit(mma_done);
      volatile int never = 0;
      mbar_wait(mma_done, 0, &never);
    }
  } else {
    // ================= softmax / epilogue (warps 2..5) =================
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // query row within the tile = TMEM lane
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    const float c = a.scale_log2;
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const uint32_t ph = j & 1;
      if (!warp_wait(s_full, ph, s_abort)) { ok = false; break; }
      tc_fence_after();
      // pass 1: row max (independent partial maxima)
      float mx[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t s0[32], s1[32];
        tmem_ld32(trow + kColS + half * 64, s0);
        tmem_ld32(trow + kColS + half * 64 + 32, s1);
        tmem_wait_ld();
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          mx[k & 7] = fmaxf(mx[k & 7], __uint_as_float(s0[k]));
          mx[k & 7] = fmaxf(mx[k & 7], __uint_as_float(s1[k]));
        }
      }
      const float mt = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_cand = fmaxf(m_run, mt * c);
      const bool grow = m_cand > m_run + kRescaleThreshold;  // always on the first tile
      const float m_use = grow ? m_cand : m_run;
      const float alpha = fast_exp2(m_run - m_use);  // 1 if kept, 0 on the first tile
      // pass 2: exponentials, row sum, bf16 packing.  s_full(j) implies that
      // PV_{j-1} is complete (the MMA warp waited for it before issuing S_j),
      // so P_j may go into the S columns already read: column t/2 holds
      // elements t, t+1 (lower index in the low half).
      float sum[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t s0[32], s1[32];
        tmem_ld32(trow + kColS + half * 64, s0);
        tmem_ld32(trow + kColS + half * 64 + 32, s1);
        tmem_wait_ld();
        uint32_t pk[32];
#pragma unroll
        for (int k = 0; k < 16; ++k) {
          const float p0 = fast_exp2(fmaf(__uint_as_float(s0[2 * k]), c, -m_use));
          const float p1 = fast_exp2(fmaf(__uint_as_float(s0[2 * k + 1]), c, -m_use));
          const float p2 = fast_exp2(fmaf(__uint_as_float(s1[2 * k]), c, -m_use));
          const float p3 = fast_exp2(fmaf(__uint_as_float(s1[2 * k + 1]), c, -m_use));
          sum[k & 3] += (p0 + p1) + (p2 + p3);
          pk[k] = pack_bf16x2(p0, p1);
          pk[16 + k] = pack_bf16x2(p2, p3);
        }
        tmem_st32(trow + kColS + half * 32, pk);
      }
      if (j > 0) {
        // O is stable (PV_{j-1} done); move it to the new max when any row of
        // the warp grew past the threshold
        if (!warp_wait(o_done, ph ^ 1, s_abort)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            tmem_ld32(trow + kColO + cc * 32, ov);
            tmem_wait_ld();
#pragma unroll
            for (int k = 0; k < 32; ++k) ov[k] = __float_as_uint(__uint_as_float(ov[k]) * alpha);
            tmem_st32(trow + kColO + cc * 32, ov);
          }
        }
      }
      tmem_wait_st();
      l = l * alpha + ((sum[0] + sum[1]) + (sum[2] + sum[3]));
      m_run = m_use;
      tc_fence_before();
      mbar_arrive(p_full);
    }
    // epilogue
    uint16_t *orow = a.O + ((size_t)row * BM + r) * D;
    bool have = ok && n > 0;
    if (have) have = mbar_wait(o_done, (n - 1) & 1, s_abort);
    // tcgen05.ld is warp-collective: decide once for the whole warp
    const bool good = __all_sync(0xffffffffu, have && !*s_abort);
    tc_fence_after();
    const float inv = good ? 1.0f / l : 0.f;
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t ov[32];
      if (good) {
        tmem_ld32(trow + kColO + cc * 32, ov);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int k = 0; k < 32; ++k) ov[k] = 0u;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 v;
        v.x = pack_bf16x2(__uint_as_float(ov[8 * q + 0]) * inv, __uint_as_float(ov[8 * q + 1]) * inv);
        v.y = pack_bf16x2(__uint_as_float(ov[8 * q + 2]) * inv, __uint_as_float(ov[8 * q + 3]) * inv);
        v.z = pack_bf16x2(__uint_as_float(ov[8 * q + 4]) * inv, __uint_as_float(ov[8 * q + 5]) * inv);
        v.w = pack_bf16x2(__uint_as_float(ov[8 * q + 6]) * inv, __uint_as_float(ov[8 * q + 7]) * inv);
        *reinterpret_cast<uint4 *>(orow + cc * 32 + q * 8) = v;
      }
    }
    if (a.lse) a.lse[(size_t)row * BM + r] = good ? (m_run + __log2f(l)) * 0.69314718055994531f : -INFINITY;
  }

  if (*s_abort && threadIdx.x == 0) flag_error(a.dev_status, VELOX_DEV_WAIT_TIMEOUT);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [H][rows][128] bf16 as a 3-D map (channel, token, head), 64 x 128 boxes.
bool make_map(CUtensorMap *map, const void *ptr, int rows, int H) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)H};
  cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)rows * D * 2};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

int attn_max_route() { return kMaxRoute; }

cudaError_t launch_attn(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                        const int32_t *route_ids, const int32_t *route_len, int R_max, int H,
                        int N, int M, float softmax_scale, uint16_t *O, float *lse,
                        int32_t *dev_status, cudaStream_t stream, bool *map_failed) {
  *map_failed = false;
  CUtensorMap mq, mk, mv;
  if (!make_map(&mq, Q, N * BM, H) || !make_map(&mk, K, M * BN, H) ||
      !make_map(&mv, V, M * BN, H)) {
    *map_failed = true;
    return cudaErrorInvalidValue;
  }
  AttnArgs a;
  a.route_ids = route_ids;
  a.route_len = route_len;
  a.R_max = R_max;
  a.N = N;
  a.M = M;
  a.scale_log2 = softmax_scale * 1.4426950408889634f;
  a.O = O;
  a.lse = lse;
  a.dev_status = dev_status;
  // dynamic tail: route list (uint16 x R_max, 16-byte rounded), id bitmap
  uint32_t list_bytes = route_ids ? ((uint32_t)R_max * 2u + 15u) & ~15u : 0u;
  uint32_t bits_bytes = route_ids ? (uint32_t)((M + 31) / 32) * 4u : 0u;
  a.bits_offset = kOffDyn + list_bytes;
  const size_t smem = (size_t)a.bits_offset + bits_bytes + 1024;  // + alignment slack
  cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  attn_kernel<<<H * N, kThreads, smem, stream>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace velox
